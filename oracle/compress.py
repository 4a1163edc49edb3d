"""c4a / c128a compressors (oracle side).

[P1] "c4a (the milder scheme)": each compressed entry is a weighted sum of 8
uncompressed states, the next entry shifted by 4.  "c128a (the aggressive
scheme)": a weighted sum of 128 states at stride 128.  [P2] Step 4 shows
C4A[1] mixing S0..S7, C4A[2] mixing S4..S11, C128A[0] = S0..S127 and
C128A[1] = S128..S255.

Reading adopted (it reproduces all four diagram examples):
* entry i of stride s with K taps mixes positions s*i + s - K + j, j < K
  (c4a: [4i-4, 4i+4); c128a: [128i, 128i+128)); taps at a position < 0 are
  zero and the weights are not renormalised;
* entries exist only for stride blocks [s*i, s*i+s) lying wholly before the
  uncompressed window: N = max(0, floor((t - W) / s));
* states are mixed un-rotated and the entry is then rotated at its block's
  first position pos0 + s*i (``pos0`` = position of raw row 0);
* w[j][c] are per-tap, per-channel weights (the CUDA side receives them as
  fp32 and so does this function).
"""
from __future__ import annotations

import numpy as np

from .rope import rope


def n_entries(t: int, window: int, stride: int) -> int:
    return max(0, (t - window) // stride)


def tap_positions(i: int, stride: int, k_taps: int) -> np.ndarray:
    return stride * i + stride - k_taps + np.arange(k_taps)


def compress(s_raw, w, stride: int, window: int, pos0: int = 0,
             rope_dim: int = 64, base: float = 10000.0) -> np.ndarray:
    """s_raw [t][D] (float64), w [K][D] -> entries [N][D] float64 (unrounded)."""
    s_raw = np.asarray(s_raw, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    t, d = s_raw.shape
    k_taps = w.shape[0]
    n = n_entries(t, window, stride)
    out = np.zeros((n, d), dtype=np.float64)
    i = np.arange(n)
    for j in range(k_taps):
        p = stride * i + stride - k_taps + j
        live = p >= 0
        out[live] += w[j][None, :] * s_raw[p[live]]
    return rope(out, pos0 + stride * i, rope_dim, base)


def append_state(s_hist, w, stride: int, window: int, rope_dim: int = 64, base: float = 10000.0):
    """Incremental maintenance of one layer's caches for a decode step (the
    steps either side of the path, [P1] "compressor-state blocks"): after the
    state of position t = len(s_hist) - 1 is appended, the caches hold
      * the window: rope(S[p], p) for p in [max(0, t + 1 - W), t + 1);
      * the compressed entries 0 .. n_entries(t + 1, W, s) - 1, each exactly
        the entry `compress` makes from the whole history.
    Reading: appending token by token must reach the same caches as
    compressing the whole history at once; an entry is emitted the step its
    stride block leaves the window.  s_hist [t+1][D] float64 (unrotated),
    w [K][D].  Returns (window positions, window rows [.][D], entries [N][D])."""
    s_hist = np.asarray(s_hist, dtype=np.float64)
    t1 = s_hist.shape[0]
    pos = np.arange(max(0, t1 - window), t1)
    win = np.stack([rope(s_hist[p], int(p), rope_dim, base) for p in pos]) if len(pos) else np.zeros((0, s_hist.shape[1]))
    ent = compress(s_hist, w, stride, window, 0, rope_dim, base)
    return pos, win, ent
