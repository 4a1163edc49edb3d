"""Shared-K/V decode attention with inverse RoPE on the output (oracle side).

[P2] Step 3: one cached vector S_j per token is compared with the query
(score = Q_i . S_j) and mixed into the output as content; Step 1 gives the
softmax-weighted sum.  [P1] "The sliding window": every layer also reads a
128-token uncompressed window.  [P1] "Shared key and value": an inverse RoPE is
applied to the attention output.  [P1] "c4a" / "c128a" and [P2] Step 5: c4a
reads the selected compressed entries, c128a reads all of them.

Reading adopted: one softmax over the union of the read compressed rows and
the window rows, scale 1/sqrt(D) unless given; the query arrives already
rotated at its position t, and the output's rotary channels are rotated by -t.
"""
from __future__ import annotations

import numpy as np

from .rope import rope


def attend(q, k, v, scale: float) -> np.ndarray:
    """General softmax attention, q [H][D], k [R][D], v [R][Dv] -> [H][Dv]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * (q @ k.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v


def shared_kv_decode(q, rows, scale: float, t: int, rope_dim: int = 64,
                     base: float = 10000.0) -> np.ndarray:
    """One decode query block over rows that serve as both keys and values."""
    o = attend(q, rows, rows, scale)
    return rope(o, -t, rope_dim, base)


def sparse_decode(q, comp_rows, win_rows, idx, t: int, scale: float,
                  rope_dim: int = 64, base: float = 10000.0) -> np.ndarray:
    """Batched c4a decode.

    q [B][H][D]; comp_rows [B][N][D] (dequantised); win_rows [B][W][D];
    idx [B][k] (ascending, -1 padded) -> out [B][H][D] float64.
    """
    out = []
    for b in range(len(q)):
        sel = np.asarray(idx[b])
        sel = sel[sel >= 0]
        rows = np.concatenate([np.asarray(comp_rows[b])[sel], np.asarray(win_rows[b])], axis=0)
        out.append(shared_kv_decode(q[b], rows, scale, t, rope_dim, base))
    return np.stack(out)


def dense_decode(q, comp_rows, win_rows, t: int, scale: float,
                 rope_dim: int = 64, base: float = 10000.0) -> np.ndarray:
    """Batched c128a decode over all compressed entries plus the window."""
    out = []
    for b in range(len(q)):
        rows = np.concatenate([np.asarray(comp_rows[b]), np.asarray(win_rows[b])], axis=0)
        out.append(shared_kv_decode(q[b], rows, scale, t, rope_dim, base))
    return np.stack(out)
