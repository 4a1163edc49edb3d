"""Number formats of the caches: bf16, fp8 E4M3, fp4 E2M1 (oracle side).

Definitions:
* bf16: the top 16 bits of an IEEE binary32.
* E4M3 (OCP 8-bit floating point spec, "E4M3"): 1 sign, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); no
  infinities; S.1111.111 is NaN; largest finite magnitude 448.
* E2M1 (OCP Microscaling spec, FP4 "E2M1"): 1 sign, 2 exponent bits with bias
  1, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no inf/NaN.

Quantisers follow the cache formats the pages name (fp8 attention cache with
a per-token scale, [P1] quantisation paragraphs; fp4 E2M1 with one E4M3 scale
per 16 channels, [P3] "storing the main KV in FP4").  The pages give no
rounding rule; the reading used here (and fixed for the CUDA side too) is:

* fp8 row:  amax = max|x| (fp32), scale = fp32(amax / 448) (IEEE fp32
  division; 1.0 when amax == 0), code = E4M3(fp32(x / scale)) with round to
  nearest even and saturation to +-448.
* fp4 group of 16: amax (fp32), scale code = E4M3(fp32(amax / 6)) (nearest
  even, saturating), s = value of that code; code = E2M1(fp32(x / s)) nearest
  even, saturating to +-6; all codes 0 when s == 0.  Nibbles are packed two
  per byte, the even channel in the low nibble.
* The sign of a value that rounds to zero is kept (IEEE conversion rule).
* fp8 with bf16 rotary channels (the layout [P1] describes for the attention
  cache: "fp8 for most dimensions", the RoPE dimensions kept in bf16): the
  first D - 64 channels of a row are quantised as an fp8 row (amax, scale and
  codes over those channels only); the last 64 (rotary) channels are stored as
  bf16 (nearest even from fp32 input, unchanged bits from bf16 input).  A row
  is D - 64 code bytes followed by the 64 bf16 values (little-endian, 128
  bytes), D + 64 bytes in all, plus the fp32 scale.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------- bf16
def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 to the nearest bf16 (ties to even), directly (one rounding)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    ax = np.abs(x)
    tiny = ax < 2.0 ** -126
    # normal range: 8 significant bits
    m, e = np.frexp(np.where(tiny, 1.0, x))
    out = np.ldexp(np.rint(m * 256.0), e - 8)
    # subnormal range: fixed spacing 2^-133
    sub = np.rint(x / 2.0 ** -133) * 2.0 ** -133
    out = np.where(tiny, sub, out)
    out = np.where(np.abs(out) > 3.3895313892515355e38, np.copysign(np.inf, x), out)
    return (out.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def round_bf16(x) -> np.ndarray:
    return bf16_bits_to_f64(f64_to_bf16_bits(x))


# ----------------------------------------------------------------- E4M3
def _e4m3_value(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (1 - 7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
E4M3_MAX = 448.0


def _e2m1_value(code: int) -> float:
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * (m / 2.0)
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
E2M1_MAX = 6.0


def _encode_nearest_even(v: np.ndarray, pos_values: np.ndarray, sign_bit: int) -> np.ndarray:
    """Encode |v| to the nearest of ``pos_values`` (codes 0..n-1, increasing),
    ties to the even code, saturating at the largest; sign bit from v."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    n = len(pos_values)
    hi = np.searchsorted(pos_values, a, side="left")        # first value >= a
    hi = np.clip(hi, 0, n - 1)
    lo = np.clip(hi - 1, 0, n - 1)
    d_lo = a - pos_values[lo]
    d_hi = pos_values[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= pos_values[-1], n - 1, code)        # saturate
    code = np.where(a == pos_values[hi], hi, code)           # exact hits
    neg = np.signbit(v)
    return (code | np.where(neg, sign_bit, 0)).astype(np.uint8)


_E4M3_POS = E4M3_TABLE[:0x7F]          # codes 0x00..0x7E, 0 .. 448
_E2M1_POS = E2M1_TABLE[:8]             # codes 0..7, 0 .. 6


def e4m3_encode(v) -> np.ndarray:
    return _encode_nearest_even(v, _E4M3_POS, 0x80)


def e2m1_encode(v) -> np.ndarray:
    return _encode_nearest_even(v, _E2M1_POS, 0x8)


# ----------------------------------------------------------------- quantisers
def quantize_fp8_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """fp32 rows [R][D] -> (codes u8 [R][D], scales f32 [R])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = (x / scale[..., None]).astype(np.float32)
    return e4m3_encode(q), scale


def quantize_fp4_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """fp32 rows [R][D] -> (packed codes u8 [R][D/2], E4M3 scale codes u8 [R][D/16])."""
    x = np.asarray(x, dtype=np.float32)
    r, d = x.shape
    g = x.reshape(r, d // 16, 16)
    amax = np.max(np.abs(g), axis=-1)
    sc_code = e4m3_encode((amax / np.float32(6.0)).astype(np.float32))
    s = E4M3_TABLE[sc_code].astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = (g / safe[..., None]).astype(np.float32)
    nib = np.where((s > 0)[..., None], e2m1_encode(q), 0).astype(np.uint8).reshape(r, d)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, sc_code.astype(np.uint8)


def dequant_fp8_rows(codes, scales) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)] * np.asarray(scales, dtype=np.float64)[..., None]


def unpack_fp4(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def dequant_fp4_rows(codes, scale_codes) -> np.ndarray:
    nib = unpack_fp4(codes)
    vals = E2M1_TABLE[nib]
    sc = E4M3_TABLE[np.asarray(scale_codes, dtype=np.uint8)]
    return vals * np.repeat(sc, 16, axis=-1)


ROPE_BF16_CHANNELS = 64  # rotary channels kept in bf16 by the fp8 + bf16-rotary layout


def quantize_fp8_rope_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """fp32 rows [R][D] -> (row bytes u8 [R][D + 64], scales f32 [R]): the
    first D - 64 channels as fp8 codes under one scale from their own amax,
    then the last 64 channels as bf16 (2 bytes each, little-endian)."""
    x = np.asarray(x, dtype=np.float32)
    r, d = x.shape
    nr = d - ROPE_BF16_CHANNELS
    body = x[:, :nr]
    amax = np.max(np.abs(body), axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    codes = e4m3_encode((body / scale[..., None]).astype(np.float32))
    rope = f64_to_bf16_bits(x[:, nr:].astype(np.float64)).astype("<u2").view(np.uint8).reshape(r, 2 * ROPE_BF16_CHANNELS)
    return np.concatenate([codes, rope], axis=1), scale


def dequant_fp8_rope_rows(row_bytes, scales) -> np.ndarray:
    """Row bytes u8 [R][D + 64] + scales f32 [R] -> float64 [R][D]."""
    b = np.ascontiguousarray(np.asarray(row_bytes, dtype=np.uint8))
    d = b.shape[-1] - ROPE_BF16_CHANNELS
    nr = d - ROPE_BF16_CHANNELS
    body = E4M3_TABLE[b[..., :nr]] * np.asarray(scales, dtype=np.float64)[..., None]
    rope = bf16_bits_to_f64(np.ascontiguousarray(b[..., nr:]).view("<u2"))
    return np.concatenate([body, rope], axis=-1)


FMT_BF16, FMT_FP8, FMT_FP4, FMT_FP8_ROPE_BF16 = 0, 1, 2, 3


def dequant(fmt: int, codes, scales=None) -> np.ndarray:
    """Rows of any cache format as float64."""
    if fmt == FMT_BF16:
        return bf16_bits_to_f64(codes)
    if fmt == FMT_FP8:
        return dequant_fp8_rows(codes, scales)
    if fmt == FMT_FP4:
        return dequant_fp4_rows(codes, scales)
    if fmt == FMT_FP8_ROPE_BF16:
        return dequant_fp8_rope_rows(codes, scales)
    raise ValueError(f"unknown format {fmt}")
