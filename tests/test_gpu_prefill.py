"""The skewed prefill workload: T = 32768 tokens at the DeepSeek-V3 shape with a
Zipf(1.1) per-expert router-logit offset (initial max/mean load ~20), run for 20
consecutive steps, each followed by the bias update (gamma = 0.001) that feeds
back into the next step's routing.  Steps 0 and 19 are checked against the
oracle on 16 sampled tokens each."""
import numpy as np
import pytest
import torch

import synth
from tests._util import np_
from tests.test_gpu_layer import build_layer, check_layer_against_oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_prefill_skewed_twenty_bias_steps(lib):
    s = synth.PREFILL
    T, E, K = s.T, s.E, s.K
    off = synth.zipf_offset(E, synth.zipf_kappa_default(), synth.seed_of(s, synth.ZIPF))
    layer, master, wr, b = build_layer(lib, s, device="cuda", offset=off)
    gamma = 0.001
    loads, biases = [], [np_(layer.e_bias).copy()]
    for step in range(20):
        x = synth.activations(T, s.H, synth.seed_of(s, synth.X) + 1000 * step, s.x_outlier_frac, device="cuda")
        layer.forward(x)
        torch.cuda.synchronize()
        if step in (0, 19):
            # 16 sampled tokens and 16 shared-expert rows against the oracle, routed
            # with this step's bias (the bias the previous steps' updates produced)
            check_layer_against_oracle(layer, s, x, wr, biases[step], n_tokens=16, seed=3 + step, offset=off,
                                       segments=False, n_shared_rows=16)
        layer.bias_update(gamma)
        torch.cuda.synchronize()
        loads.append(np_(layer.load).copy())
        biases.append(np_(layer.e_bias).copy())
        assert np.array_equal(np_(layer.offsets), np.concatenate([[0], np.cumsum(loads[-1])]))
    assert int(layer.status.item()) == 0
    g32 = np.float32(gamma)
    for st in range(20):
        load = loads[st].astype(np.int64)
        assert load.sum() == T * K
        # the update moved every bias by exactly +gamma, -gamma or 0, by the sign of mean - load
        sign = np.sign(T * K - E * load)
        want = np.where(sign > 0, (biases[st] + g32).astype(np.float32),
                        np.where(sign < 0, (biases[st] - g32).astype(np.float32), biases[st]))
        assert np.array_equal(biases[st + 1], want)
    ratio = [l.max() / l.mean() for l in loads]
    assert ratio[0] > 10                       # the workload is skewed
    assert ratio[-1] < ratio[0]                # and the bias pulls the loads together
