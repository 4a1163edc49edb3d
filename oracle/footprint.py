"""Closed-form KV-cache footprints (oracle side).

[P1] opening summary and "Key points": about 9.62 GiB of bf16 KV per 1M-token
sequence for the 61-layer hybrid stack, versus about 83.9 GiB for a V3.2-style
stack, about 8.7x smaller; fp8 attention plus fp4 indexer caches cut roughly
another 2x.  [P1] "To judge the saving": 1408 B per token per layer (576 MLA
values + 128 indexer values, bf16) over 61 layers.  [P1] hybrid cache manager
paragraph: about 320 MiB per c4a layer and about 8 MiB per c128a layer at 1M.
[P1] "c128a": at most about 8,000 compressed entries at 1M.

Geometry used (the pages give 128 indexer values, 61 = 30 c4a + 31 c128a
layers and a 128-token window; the 512-dim shared state is the spec's): a c4a
layer stores N4 = floor((T-W)/4) entries of 512 + 128 values plus W window rows
of 512 values; a c128a layer stores N128 = floor((T-W)/128) entries of 512
values plus the window.  "1M" is 2^20 tokens.
"""
from __future__ import annotations

from .compress import n_entries

MIB = 2 ** 20
GIB = 2 ** 30


def layer_bytes(kind: str, t: int, d: int = 512, di: int = 128, window: int = 128,
                main_fmt: str = "bf16", index_fmt: str = "bf16") -> int:
    """Bytes of one layer's cache for one sequence at context t."""
    def row_bytes(fmt: str, n: int) -> int:
        if fmt == "bf16":
            return 2 * n
        if fmt == "fp8":          # codes + one fp32 scale per row
            return n + 4
        if fmt == "fp4":          # two codes per byte + one E4M3 byte per 16
            return n // 2 + n // 16
        raise ValueError(fmt)

    if kind == "c4a":
        n = n_entries(t, window, 4)
        return n * (row_bytes(main_fmt, d) + row_bytes(index_fmt, di)) + window * row_bytes(main_fmt, d)
    if kind == "c128a":
        n = n_entries(t, window, 128)
        return n * row_bytes(main_fmt, d) + window * row_bytes(main_fmt, d)
    raise ValueError(kind)


def stack_bytes(t: int, n_c4a: int = 30, n_c128a: int = 31, **kw) -> int:
    return n_c4a * layer_bytes("c4a", t, **kw) + n_c128a * layer_bytes("c128a", t, **kw)


def v32_stack_bytes(t: int, layers: int = 61, mla: int = 576, di: int = 128) -> int:
    return (mla + di) * 2 * t * layers
