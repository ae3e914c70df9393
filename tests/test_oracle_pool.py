"""The process pool the full-size GPU parity tests use for the oracle's expert
FFNs returns exactly what calling the oracle directly returns (CPU only)."""
import numpy as np

import oracle
import synth
from tests import _oracle_pool


def test_pool_matches_direct_oracle():
    s = synth.TINY
    x = synth.activations(5, s.H, 3).float().numpy()
    xq, xs = oracle.quant_1x128(x)
    got = _oracle_pool.expert_outputs(s, {2: (xq[:3], xs[:3]), -1: (xq, xs)}, device="cpu")
    for e, rows in ((2, slice(0, 3)), (-1, slice(0, 5))):
        tid13, tid2 = (synth.SH13, synth.SH2) if e < 0 else (synth.W13, synth.W2)
        w13 = synth.expert_weight(2 * s.I, s.H, s.w_std, synth.seed_of(s, tid13, max(e, 0))).float().numpy()
        w2 = synth.expert_weight(s.H, s.I, s.w_std, synth.seed_of(s, tid2, max(e, 0))).float().numpy()
        q13, s13 = oracle.quant_128x128(w13)
        q2, s2 = oracle.quant_128x128(w2)
        y16, _ = oracle.expert_ffn(xq[rows], xs[rows], q13, s13, q2, s2)
        assert np.array_equal(got[e], y16.astype(np.float32))
