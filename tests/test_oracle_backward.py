"""Pins of the oracle's backward FP8 GEMMs (dgrad, wgrad) and the 128x1 quantiser."""
import numpy as np

import oracle
import synth
from oracle.backward import dgrad_blockscaled, quant_128x1, wgrad_blockscaled


def _int_codes(shape, seed, hi=8):
    """E4M3 codes of small signed integers (exact in e4m3) and their values."""
    rng = np.random.default_rng(seed)
    v = rng.integers(-hi, hi + 1, size=shape).astype(np.float32)
    return oracle.e4m3_encode(v), v.astype(np.int64)


def test_quant_128x1_is_the_transposed_1x128_tiling():
    x = synth.activations(256, 384, 11).float().numpy()
    q, s, rows = quant_128x1(x, [0, 256])
    qt, st = oracle.quant_1x128(x.T)
    assert list(rows) == [0, 128, 256]
    assert np.array_equal(q, qt.T) and np.array_equal(s, st.T)


def test_quant_128x1_tiles_stop_at_group_boundaries():
    x = np.ones((300, 128), dtype=np.float32)
    x[129, 5] = 1000.0                      # in group 0's second (2-row) tile
    q, s, rows = quant_128x1(x, [0, 130, 130, 300])
    assert list(rows) == [0, 128, 130, 258, 300]
    assert s[1, 5] == np.float32(np.float32(1000.0) / np.float32(448.0))
    assert s[2, 5] == np.float32(np.float32(1.0) / np.float32(448.0))    # group 2 unaffected
    # every tile decodes back to its values within one e4m3 step
    deq = np.zeros_like(x, dtype=np.float64)
    for t in range(len(rows) - 1):
        deq[rows[t]:rows[t + 1]] = oracle.e4m3_decode(q[rows[t]:rows[t + 1]]) * s[t][None, :].astype(np.float64)
    assert np.allclose(deq, x, rtol=2 ** -3)


def test_dgrad_integer_exact():
    dyq, dyv = _int_codes((40, 256), 1)
    wq, wv = _int_codes((256, 384), 2)
    sdy = np.ones((40, 2), np.float32)
    sw = np.ones((2, 3), np.float32)
    got = dgrad_blockscaled(dyq, sdy, wq, sw)
    assert np.array_equal(got, (dyv @ wv).astype(np.float64))


def test_dgrad_equals_product_of_dequantised_operands():
    dy = synth.activations(70, 384, 3).float().numpy()
    w = synth.normal((384, 256), 0.02, 4).numpy()
    dyq, sdy = oracle.quant_1x128(dy)
    wq, sw = oracle.quant_128x128(w)
    got = dgrad_blockscaled(dyq, sdy, wq, sw)
    want = oracle.dequant_1x128(dyq, sdy) @ oracle.dequant_128x128(wq, sw)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # scales enter per (row, 128 of N) and per (128 of N, 128 of K): doubling one block's scale
    sw2 = sw.copy()
    sw2[1, 0] *= 2
    d = dgrad_blockscaled(dyq, sdy, wq, sw2) - got
    assert np.allclose(d[:, 128:], 0) and not np.allclose(d[:, :128], 0)


def test_wgrad_per_group_equals_product_of_dequantised_tiles():
    offs = [0, 200, 200, 330]
    dy = synth.activations(330, 256, 5).float().numpy()
    x = synth.activations(330, 128, 6).float().numpy()
    dyq, sdy, rows = quant_128x1(dy, offs)
    xq, sx, rows_x = quant_128x1(x, offs)
    assert np.array_equal(rows, rows_x)

    def deq(q, s):
        out = np.zeros(q.shape)
        for t in range(len(rows) - 1):
            out[rows[t]:rows[t + 1]] = oracle.e4m3_decode(q[rows[t]:rows[t + 1]]) * s[t][None, :].astype(np.float64)
        return out

    D, X = deq(dyq, sdy), deq(xq, sx)
    for g in range(3):
        r0, r1 = offs[g], offs[g + 1]
        got = wgrad_blockscaled(dyq, sdy, xq, sx, rows, r0, r1)
        want = D[r0:r1].T @ X[r0:r1]
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * max(np.abs(want).max(), 1.0))
    # an empty group gives zero
    assert not wgrad_blockscaled(dyq, sdy, xq, sx, rows, 200, 200).any()


def test_wgrad_integer_exact():
    dyq, dyv = _int_codes((256, 128), 7)
    xq, xv = _int_codes((256, 256), 8)
    ones_dy = np.ones((2, 128), np.float32)
    ones_x = np.ones((2, 256), np.float32)
    got = wgrad_blockscaled(dyq, ones_dy, xq, ones_x, np.array([0, 128, 256]), 0, 256)
    assert np.array_equal(got, (dyv.T @ xv).astype(np.float64))
