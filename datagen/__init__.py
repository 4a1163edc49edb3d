"""Seeded, counter-based synthetic input generator.

This module is the only code that both the float64 oracle and the CUDA path
consume.  It holds none of the method's arithmetic: it only produces input
bytes (raw shared states, cache rows, queries, indexer keys and queries,
compression weights) from a seed, so that both sides read identical inputs.

Generator definition (the CUDA twin in ``datagen/csrc/datagen.cu`` implements
the same integer recipe, so both produce bit-identical bytes):

* ``mix64`` is the SplitMix64 output function (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31``.
* A stream key is ``mix64(mix64(seed + GOLDEN) ^ mix64(tensor_id * GOLDEN2 + layer))``.
* Draw ``i`` of a stream is ``mix64(key + (i + 1) * GOLDEN)`` (wrapping uint64).
* A "normal" element with flat index ``e`` uses draws ``3e, 3e+1, 3e+2``; each
  64-bit draw is split into four 16-bit integers ``u`` (low half first).  The
  value is ``(sum of the twelve u - 393210) / 65536``: the Irwin-Hall sum of
  twelve U(0,1) minus 6, a textbook approximate N(0,1) with unit variance.
  The numerator has at most 19 significant bits, so the value is exact in
  float32 and is then rounded once to bfloat16 (round to nearest even).
* A uniform integer in ``[lo, hi]`` with flat index ``e`` is
  ``lo + ((draw_e >> 32) * (hi - lo + 1) >> 32)``.

No transcendental function is evaluated on either side, so there is no
last-ulp disagreement between host and device generators.
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
GOLDEN2 = np.uint64(0xD1B54A32D192ED03)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# Tensor ids: which synthetic tensor a stream feeds.
TID_RAW_S = 1          # raw shared states S [B][t][D] (bf16, ~N(0,1))
TID_W_LOGITS = 2       # compression weight logits [K][D] (f64 -> softmax -> fp32)
TID_COMP = 3           # compressed cache rows [B][N][D] (bf16, ~N(0,1))
TID_WIN = 4            # window cache rows [B][W][D] (bf16, ~N(0,1))
TID_QIDX = 5           # indexer queries [B][Di] (integers in [-8, 8])
TID_KIDX = 6           # indexer keys [B][N][Di] (integers in [-8, 8])
TID_Q = 7              # attention queries [B][H][D] (bf16, ~N(0,1))
TID_KIDX_FP4 = 8       # fp4 indexer key codes [B][N][Di]
TID_STATES = 9         # states to quantise [rows][D] (bf16, ~N(0,1))


def _py_mix64(z: int) -> int:
    z &= _MASK64
    z ^= z >> 30
    z = (z * 0xBF58476D1CE4E5B9) & _MASK64
    z ^= z >> 27
    z = (z * 0x94D049BB133111EB) & _MASK64
    z ^= z >> 31
    return z


def stream_key(seed: int, tensor_id: int, layer: int = 0) -> int:
    """64-bit key of the stream for (seed, tensor_id, layer)."""
    a = _py_mix64((seed + 0x9E3779B97F4A7C15) & _MASK64)
    b = _py_mix64((tensor_id * 0xD1B54A32D192ED03 + layer) & _MASK64)
    return _py_mix64(a ^ b)


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = z ^ (z >> np.uint64(30))
        z = z * _M1
        z = z ^ (z >> np.uint64(27))
        z = z * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def draws(key: int, counters: np.ndarray) -> np.ndarray:
    """Draws ``counters`` (uint64 array) of stream ``key``."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (c + np.uint64(1)) * GOLDEN
    return _mix64(z)


def _f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 bits (nearest, ties to even)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    b = b + np.uint64(0x7FFF) + lsb
    return (b >> np.uint64(16)).astype(np.uint16)


def normal_values(key: int, flat_index: np.ndarray) -> np.ndarray:
    """Irwin-Hall(12) - 6 values (float64, exact) for the given flat indices."""
    e = np.asarray(flat_index, dtype=np.uint64)
    total = np.zeros(e.shape, dtype=np.int64)
    for j in range(3):
        d = draws(key, e * np.uint64(3) + np.uint64(j))
        for s in (0, 16, 32, 48):
            total += ((d >> np.uint64(s)) & np.uint64(0xFFFF)).astype(np.int64)
    return (total - 393210).astype(np.float64) / 65536.0


def normal_bf16(key: int, count: int, offset: int = 0) -> np.ndarray:
    """``count`` consecutive bf16 (uint16 bits) ~N(0,1) values from ``offset``."""
    idx = np.arange(offset, offset + count, dtype=np.uint64)
    return _f32_to_bf16_bits(normal_values(key, idx).astype(np.float32))


def normal_bf16_at(key: int, flat_index: np.ndarray) -> np.ndarray:
    """bf16 bits of the normal elements at arbitrary flat indices."""
    return _f32_to_bf16_bits(normal_values(key, flat_index).astype(np.float32))


def uniform_int_at(key: int, flat_index: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """Uniform integers in [lo, hi] (int64) at the given flat indices."""
    d = draws(key, np.asarray(flat_index, dtype=np.uint64))
    span = np.uint64(hi - lo + 1)
    with np.errstate(over="ignore"):
        v = ((d >> np.uint64(32)) * span) >> np.uint64(32)
    return v.astype(np.int64) + lo


def uniform_int(key: int, count: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    return uniform_int_at(key, np.arange(offset, offset + count, dtype=np.uint64), lo, hi)


def int_bf16(key: int, count: int, lo: int = -8, hi: int = 8, offset: int = 0) -> np.ndarray:
    """Uniform integers in [lo, hi] stored as bf16 bits (exact for |v| <= 256)."""
    v = uniform_int(key, count, lo, hi, offset).astype(np.float32)
    return _f32_to_bf16_bits(v)


def int_bf16_at(key: int, flat_index: np.ndarray, lo: int = -8, hi: int = 8) -> np.ndarray:
    return _f32_to_bf16_bits(uniform_int_at(key, flat_index, lo, hi).astype(np.float32))


# fp4 indexer keys in the quantised domain: one draw v in [0, 13] per channel,
# magnitude code v % 7 (E2M1 codes 0..6 = 0, .5, 1, 1.5, 2, 3, 4), sign v // 7.
# Every group of 16 channels carries the E4M3 scale code 0x40 (= 2.0).
FP4_INDEX_SCALE_CODE = 0x40


def fp4_index_nibbles_at(key: int, flat_index: np.ndarray) -> np.ndarray:
    v = uniform_int_at(key, flat_index, 0, 13)
    return ((v // 7) << 3 | (v % 7)).astype(np.uint8)


def fp4_index_keys_rows(key: int, rows: np.ndarray, di: int) -> tuple[np.ndarray, np.ndarray]:
    """Codes [len(rows)][di/2] (low nibble = even channel) and scales [len(rows)][di/16]."""
    rows = np.asarray(rows, dtype=np.uint64)
    flat = rows[:, None] * np.uint64(di) + np.arange(di, dtype=np.uint64)[None, :]
    nib = fp4_index_nibbles_at(key, flat.reshape(-1)).reshape(len(rows), di)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((len(rows), di // 16), FP4_INDEX_SCALE_CODE, dtype=np.uint8)
    return codes, scales


def rows_normal_bf16(key: int, rows: np.ndarray, d: int) -> np.ndarray:
    """bf16 bits [len(rows)][d] of the rows ``rows`` of a row-major [*][d] tensor."""
    rows = np.asarray(rows, dtype=np.uint64)
    flat = rows[:, None] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :]
    return normal_bf16_at(key, flat.reshape(-1)).reshape(len(rows), d)


def rows_int_bf16(key: int, rows: np.ndarray, d: int, lo: int = -8, hi: int = 8) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint64)
    flat = rows[:, None] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :]
    return int_bf16_at(key, flat.reshape(-1), lo, hi).reshape(len(rows), d)


def compress_weights(seed: int, layer: int, k_taps: int, d: int) -> np.ndarray:
    """Per-position, per-channel softmax-normalised weights [K][D] as float32.

    Logits are ~N(0,1) (the normal recipe above, kept in float64); each
    channel's K logits are normalised by a softmax over the tap axis in
    float64 and then rounded to float32.  These stand in for learned weights.
    """
    key = stream_key(seed, TID_W_LOGITS, layer)
    logits = normal_values(key, np.arange(k_taps * d, dtype=np.uint64)).reshape(k_taps, d)
    e = np.exp(logits - logits.max(axis=0, keepdims=True))
    return (e / e.sum(axis=0, keepdims=True)).astype(np.float32)
