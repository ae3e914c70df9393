"""E4M3 encoding, bf16 rounding and the two block quantisers (oracle).

Test infrastructure only (see the package docstring).

E4M3 follows the OCP OFP8 definition: 1 sign bit, 4 exponent bits with bias
7, 3 mantissa bits; no infinities; the single NaN pattern per sign is
S.1111.111; the largest finite magnitude is 1.75 * 2^8 = 448; subnormals
are M * 2^-9 for M = 1..7.  Encoding rounds to nearest, ties to even, and
saturates finite values beyond 448 to +-448 ("satfinite").

Quantisation follows [report-walkthrough] section 4.3 and [repro-guide]
section 3 (input_quant_granularity tile_wise_1x128, weight_quant_granularity
block_wise_128x128, format e4m3) and [infra-answer] (E4M3 everywhere, per-tile
1x128 and per-group 128x128): one scale per 1x128 tile of an activation row
and per 128x128 block of a weight.  The pages do not spell the scale rule
out; the reading used here is
    amax  = max |v| over the tile,
    scale = fp32(amax / 448)            (one correctly rounded fp32 division)
    q     = e4m3_rne_satfinite(fp32(v / scale))
with amax == 0 giving scale 1 and all-zero codes, and a tile holding a NaN
or an infinity giving NaN codes (0x7F) and a NaN scale.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_NAN_CODE = 0x7F


# ----------------------------------------------------------------- scalar
def e4m3_encode_scalar(v: float) -> int:
    """Encode one fp32 value as an E4M3 byte (RNE, satfinite).  Plain Python."""
    v = float(np.float32(v))
    if v != v:
        return _NAN_CODE
    sign = 0x80 if (v < 0 or (v == 0 and np.signbit(v))) else 0
    a = abs(v)
    if a >= E4M3_MAX:                      # also +-inf: saturate to the largest finite
        return sign | 0x7E
    if a < 2.0 ** -6:                      # subnormal range: multiples of 2^-9
        m = _rne(a * 2.0 ** 9)             # 0..8; 8 is exactly 2^-6, the first normal
        return sign | int(m)
    e = 0
    while a >= 2.0 ** (e + 1):
        e += 1
    while a < 2.0 ** e:
        e -= 1
    frac = a / 2.0 ** e - 1.0              # in [0, 1), exact in binary64
    q = _rne(frac * 8.0)
    if q == 8:
        e += 1
        q = 0
    code = ((e + 7) << 3) | int(q)
    if code > 0x7E:                        # cannot happen below 448, kept as a guard
        code = 0x7E
    return sign | code


def _rne(t: float) -> int:
    """Round a non-negative float to the nearest integer, ties to even."""
    f = int(np.floor(t))
    r = t - f
    if r > 0.5 or (r == 0.5 and (f & 1)):
        return f + 1
    return f


def e4m3_decode_scalar(code: int) -> float:
    """Value of one E4M3 byte (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    s = -1.0 if code & 0x80 else 1.0
    E = (code >> 3) & 0xF
    M = code & 0x7
    if E == 0xF and M == 0x7:
        return float("nan")
    if E == 0:
        return s * M * 2.0 ** -9
    return s * (1.0 + M / 8.0) * 2.0 ** (E - 7)


# ------------------------------------------------------------- vectorised
def e4m3_encode(v) -> np.ndarray:
    """Vectorised E4M3 encoder of fp32 values (same rule as the scalar one)."""
    x = np.asarray(v, dtype=np.float32).astype(np.float64)
    sign = np.where(np.signbit(x), 0x80, 0x00).astype(np.int64)
    a = np.abs(x)
    nan = np.isnan(a)
    a_ = np.where(nan, 0.0, a)
    big = a_ >= E4M3_MAX
    sub = a_ < 2.0 ** -6
    # subnormal: nearest multiple of 2^-9 (np.rint rounds half to even)
    q_sub = np.rint(a_ * 2.0 ** 9).astype(np.int64)
    # normal: a = 2^e * (1 + frac)
    safe = np.where(sub | big, 1.0, a_)
    m, ex = np.frexp(safe)                 # safe = m * 2^ex, m in [0.5, 1)
    e = ex.astype(np.int64) - 1
    frac = m * 2.0 - 1.0
    q = np.rint(frac * 8.0).astype(np.int64)
    carry = q == 8
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 0, q)
    code_n = ((e + 7) << 3) | q
    code_n = np.minimum(code_n, 0x7E)
    code = np.where(sub, q_sub, code_n)
    code = np.where(big, 0x7E, code)
    code = code | sign
    code = np.where(nan, _NAN_CODE, code)
    return code.astype(np.uint8)


_DECODE_TABLE = np.array([e4m3_decode_scalar(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """Vectorised E4M3 decoder to float64 (exact)."""
    return _DECODE_TABLE[np.asarray(codes, dtype=np.uint8)]


def round_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned
    as float64.  bf16 keeps 8 significant bits and fp32's exponent range;
    values beyond the largest finite bf16 round to +-inf, NaN stays NaN."""
    x = np.asarray(v, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    m, ex = np.frexp(np.where(fin, x, 1.0))  # x = m*2^ex, |m| in [0.5,1)
    # quantum of the 8-bit significand; below 2^-126 the bf16 grid is uniform at 2^-133
    ex_eff = np.maximum(ex, -125)
    quantum = np.ldexp(1.0, ex_eff - 8)
    r = np.rint(x / quantum) * quantum
    r = np.where(np.abs(r) > 3.3895313892515355e38, np.copysign(np.inf, x), r)
    out = np.where(fin, r, out)
    return out


# ------------------------------------------------------------ quantisers
def _quant_tiles(v32: np.ndarray):
    """Quantise rows of tiles: v32 [..., n] fp32, one scale per leading index."""
    a = np.abs(v32.astype(np.float64))
    finite = np.all(np.isfinite(a), axis=-1)
    amax = np.max(np.where(np.isfinite(a), a, 0.0), axis=-1)
    scale = np.where(amax == 0.0, np.float32(1.0),
                     (amax.astype(np.float32) / np.float32(E4M3_MAX)).astype(np.float32))
    scale = np.where(finite, scale, np.float32(np.nan)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        y = (v32 / scale[..., None]).astype(np.float32)    # fp32 division, RN
    codes = e4m3_encode(y)
    codes = np.where(finite[..., None], codes, np.uint8(_NAN_CODE)).astype(np.uint8)
    return codes, scale


def quant_1x128(x) -> tuple[np.ndarray, np.ndarray]:
    """Activation quantisation, one scale per 1x128 tile of each row.

    x: [rows, cols] values of bf16 or fp32 (cols % 128 == 0).
    Returns codes uint8 [rows, cols] and scales float32 [rows, cols/128]."""
    x32 = np.asarray(x, dtype=np.float32)
    rows, cols = x32.shape
    assert cols % 128 == 0
    codes, scale = _quant_tiles(x32.reshape(rows, cols // 128, 128))
    return codes.reshape(rows, cols), scale.reshape(rows, cols // 128)


def quant_128x128(w) -> tuple[np.ndarray, np.ndarray]:
    """Weight quantisation, one scale per 128x128 block.

    w: [rows, cols] (both % 128 == 0).  Returns codes uint8 [rows, cols] and
    scales float32 [rows/128, cols/128]."""
    w32 = np.asarray(w, dtype=np.float32)
    rows, cols = w32.shape
    assert rows % 128 == 0 and cols % 128 == 0
    blk = w32.reshape(rows // 128, 128, cols // 128, 128).transpose(0, 2, 1, 3)
    codes, scale = _quant_tiles(blk.reshape(rows // 128, cols // 128, 128 * 128))
    codes = codes.reshape(rows // 128, cols // 128, 128, 128).transpose(0, 2, 1, 3)
    return codes.reshape(rows, cols), scale


def dequant_1x128(codes, scales) -> np.ndarray:
    """decode(q) * scale per 1x128 tile, float64 (exact)."""
    v = e4m3_decode(codes)
    return v * np.repeat(np.asarray(scales, dtype=np.float64), 128, axis=1)


def dequant_128x128(codes, scales) -> np.ndarray:
    """decode(q) * scale per 128x128 block, float64 (exact)."""
    v = e4m3_decode(codes)
    s = np.asarray(scales, dtype=np.float64)
    return v * np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)
