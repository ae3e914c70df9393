"""The skewed prefill workload: T = 32768 tokens at the DeepSeek-V3 shape with a
Zipf(1.1) per-expert router-logit offset (initial max/mean load ~20), run for 20
consecutive steps, each followed by the bias update (gamma = 0.001) that feeds
back into the next step's routing."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, np_, normwise
from tests.test_gpu_kernels import check_routing, routing_tol
from tests.test_gpu_layer import _oracle_weights, build_layer

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_prefill_skewed_twenty_bias_steps(lib):
    s = synth.PREFILL
    T, E, K = s.T, s.E, s.K
    off = synth.zipf_offset(E, synth.zipf_kappa_default(), synth.seed_of(s, synth.ZIPF))
    layer, master, wr, b = build_layer(lib, s, device="cuda", offset=off)
    gamma = 0.001
    loads, biases = [], [np_(layer.e_bias).copy()]
    x0 = None
    for step in range(20):
        x = synth.activations(T, s.H, synth.seed_of(s, synth.X) + 1000 * step, s.x_outlier_frac, device="cuda")
        if step == 0:
            x0 = x
        layer.forward(x)
        if step == 0:
            out0 = layer.out.clone()
            idx0 = layer.topk_idx.clone()
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
    # step 0 against the oracle on sampled tokens (no near ties)
    xh = x0.float().cpu().numpy()
    offh = off.numpy()
    s32 = oracle.router_scores(xh, wr.cpu().numpy(), offh).astype(np.float32)
    ridx, _ = oracle.select_experts(s32, biases[0], s.n_group, s.topk_group, K, s.rho)
    same = check_routing(np_(idx0), None, ridx, s32, biases[0], s.n_group, s.topk_group, K,
                         routing_tol(xh, wr.cpu().numpy()), min_same=0.97)
    pick = np.random.default_rng(3).choice(np.where(same)[0], size=2, replace=False)
    ref = oracle.moe_forward_tokens(xh[pick], wr.cpu().numpy(), biases[0], _oracle_weights(master), s.n_group,
                                    s.topk_group, K, s.rho, offset=offh)
    assert normwise(np_(out0)[pick], ref["out"]) < TOL_NORMWISE
