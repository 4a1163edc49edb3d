"""Rotary position embedding on the last ``rope_dim`` channels (oracle side).

[P1] "Shared key and value": positions enter the shared vector through rotary
embeddings, and because the same vector is also the value, an inverse RoPE is
applied to the attention output.  The pages fix neither the pairing nor the
frequencies; the reading used here: channels (D-rope_dim+2m, D-rope_dim+2m+1)
for m < rope_dim/2 form a pair, theta_m = base^(-2m/rope_dim), base 10000,
and a pair (x, y) at position p becomes (x cos a - y sin a, x sin a + y cos a)
with a = p * theta_m.  The inverse is the same map at position -p.
"""
from __future__ import annotations

import numpy as np


def thetas(rope_dim: int = 64, base: float = 10000.0) -> np.ndarray:
    m = np.arange(rope_dim // 2, dtype=np.float64)
    return base ** (-2.0 * m / rope_dim)


def rope(x, pos, rope_dim: int = 64, base: float = 10000.0) -> np.ndarray:
    """Rotate the last ``rope_dim`` channels of x [..., D] by position ``pos``.

    ``pos`` is a scalar or an array broadcastable to x.shape[:-1].
    """
    x = np.array(x, dtype=np.float64, copy=True)
    d = x.shape[-1]
    r0 = d - rope_dim
    a = np.asarray(pos, dtype=np.float64)[..., None] * thetas(rope_dim, base)
    c, s = np.cos(a), np.sin(a)
    xe = x[..., r0 + 0::2][..., : rope_dim // 2].copy()
    xo = x[..., r0 + 1::2][..., : rope_dim // 2].copy()
    x[..., r0 + 0::2] = xe * c - xo * s
    x[..., r0 + 1::2] = xe * s + xo * c
    return x
