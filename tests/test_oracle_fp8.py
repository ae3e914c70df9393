"""Pins of the oracle's E4M3 encoder/decoder, bf16 rounding and quantisers.

Each check ties the oracle to something other than itself: hand-derived
codes from the OCP E4M3 definition (tests/golden), torch's own fp8 and bf16
conversions (library routines), exhaustive round trips and closed forms."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def test_golden_codes_scalar_and_vector():
    vals, codes = [], []
    for expr, code, _why in _rows("e4m3_codes.txt"):
        v = float(eval(expr, {"__builtins__": {}}))
        vals.append(v)
        codes.append(int(code, 16))
        assert oracle.e4m3_encode_scalar(v) == int(code, 16), expr
    got = oracle.e4m3_encode(np.array(vals, dtype=np.float32))
    assert [int(c) for c in got] == codes


def test_nan_and_inf():
    assert oracle.e4m3_encode_scalar(float("nan")) == 0x7F
    assert oracle.e4m3_encode_scalar(float("inf")) == 0x7E          # satfinite
    assert oracle.e4m3_encode_scalar(float("-inf")) == 0xFE
    assert math.isnan(oracle.e4m3_decode_scalar(0x7F))
    assert math.isnan(oracle.e4m3_decode_scalar(0xFF))


def test_decode_closed_form():
    assert oracle.e4m3_decode_scalar(0x7E) == 448.0
    assert oracle.e4m3_decode_scalar(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode_scalar(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode_scalar(0x77) == 240.0
    assert oracle.e4m3_decode_scalar(0xC4) == -3.0
    # every finite code: magnitudes strictly increase with the code
    mags = [oracle.e4m3_decode_scalar(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(mags, mags[1:]))


def test_exhaustive_round_trip():
    """decode(encode(v)) == v for all 254 finite codes (and both zeros)."""
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = oracle.e4m3_decode_scalar(c)
        assert oracle.e4m3_encode_scalar(v) == c, hex(c)
        assert int(oracle.e4m3_encode(np.array([v], dtype=np.float32))[0]) == c


def test_against_torch_float8_in_range():
    """torch.float8_e4m3fn conversion (RNE) agrees for every |v| <= 448,
    including all midpoints between neighbouring codes (the tie cases)."""
    finite = [oracle.e4m3_decode_scalar(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(finite, finite[1:])]
    rng = np.random.default_rng(0)
    rand = list(rng.uniform(-448, 448, 20000)) + list(rng.normal(0, 1e-2, 20000))
    v = np.array(finite + mids + [-m for m in mids] + rand, dtype=np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v)
    # torch keeps the sign of a value that rounds to zero; so does the oracle
    assert np.array_equal(got, ref)


def test_vector_matches_scalar_random():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 50, 3000), rng.normal(0, 1e-3, 3000),
                        rng.uniform(-600, 600, 3000)]).astype(np.float32)
    vec = oracle.e4m3_encode(v)
    for x, c in zip(v[:2000], vec[:2000]):
        assert oracle.e4m3_encode_scalar(float(x)) == int(c)


def test_round_bf16_against_torch():
    """For float32 inputs torch's fp32->bf16 conversion is a single RNE
    rounding, so it must agree with the oracle's float64->bf16 rounding."""
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    f = f[np.abs(f) < 3.38e38]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(f.astype(np.float64))
    assert np.array_equal(got, ref)


def test_quant_golden_tile():
    x = np.zeros((1, 128), dtype=np.float32)
    want = {}
    for col, val, _vs, code in _rows("quant_tile.txt"):
        x[0, int(col)] = float(val)
        want[int(col)] = int(code, 16)
    q, s = oracle.quant_1x128(x)
    assert s.shape == (1, 1) and s[0, 0] == np.float32(2.0)
    for c, code in want.items():
        assert int(q[0, c]) == code, c
    assert all(int(q[0, c]) == 0 for c in range(128) if c not in want)


def test_quant_zero_nan_and_amax_tile():
    x = np.zeros((3, 256), dtype=np.float32)
    x[1, :] = np.linspace(-3, 3, 256, dtype=np.float32)
    x[2, 5] = np.nan
    q, s = oracle.quant_1x128(x)
    assert s[0, 0] == 1.0 and s[0, 1] == 1.0 and not q[0].any()
    # the tile's amax maps to exactly +-448 (code 0x7E / 0xFE)
    assert q[1, 0] == 0xFE and q[1, 255] == 0x7E
    assert np.isnan(s[2, 0]) and np.all(q[2, :128] == 0x7F)
    assert s[2, 1] == 1.0 and not q[2, 128:].any()


def test_quant_error_bound_and_scale_rule():
    """Dequantised values are within half an E4M3 ulp (relative 2^-4) of the
    inputs for normal-range codes; scale = fp32(amax/448) exactly."""
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.normal(0, 1, (16, 512)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    q, s = oracle.quant_1x128(x)
    amax = np.abs(x.reshape(16, 4, 128)).max(-1)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    deq = oracle.dequant_1x128(q, s)
    y = x / np.repeat(s, 128, 1)
    normal = np.abs(y) >= 2 ** -6
    rel = np.abs(deq - x)[normal] / np.abs(x)[normal]
    assert rel.max() <= 2 ** -4 * (1 + 1e-6)


def test_quant_128x128_blocks():
    rng = np.random.default_rng(4)
    w = rng.normal(0, 0.02, (256, 384)).astype(np.float32)
    q, s = oracle.quant_128x128(w)
    assert q.shape == (256, 384) and s.shape == (2, 3)
    for i in range(2):
        for j in range(3):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert s[i, j] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))
            # the block's largest magnitude encodes to +-448
            r, c = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            assert int(q[i * 128 + r, j * 128 + c]) & 0x7F == 0x7E
    deq = oracle.dequant_128x128(q, s)
    assert np.abs(deq - w).max() <= np.abs(w).max() * 2 ** -4


def test_boundary_helper_matches_the_encoder():
    """The E4M3 rounding boundaries the GPU parity bands use (tests/_util) are
    exactly where the oracle's encoder changes code: just below and above every
    midpoint the codes differ, and the codes of the midpoints' neighbours agree
    with the nearest representable value."""
    from tests._util import _MIDPOINTS, e4m3_boundary_distance
    below = np.nextafter(_MIDPOINTS.astype(np.float32), np.float32(0))
    above = np.nextafter(_MIDPOINTS.astype(np.float32), np.float32(1e9))
    assert np.all(oracle.e4m3_encode(below) != oracle.e4m3_encode(above))
    assert np.all(oracle.e4m3_encode(below) + 1 == oracle.e4m3_encode(above))
    # no other code change: a fine grid between consecutive midpoints keeps one code
    rng = np.random.default_rng(0)
    for lo, hi in zip(_MIDPOINTS[:-1], _MIDPOINTS[1:]):
        v = rng.uniform(lo, hi, 64).astype(np.float32)
        v = v[(v > lo) & (v < hi)]
        assert len(set(oracle.e4m3_encode(v).tolist())) == 1
    assert e4m3_boundary_distance([1.0625])[0] == 0.0 and e4m3_boundary_distance([1.0])[0] == 0.03125   # 0.96875 and 1.0625
