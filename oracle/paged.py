"""Paged and ragged caches (oracle side; the NEXT row on per-sequence
lengths and block tables, [P1] "compressor-state blocks": the caches are
kept in blocks).

Test infrastructure: only the tests, the smoke check and the bench's CPU
baseline use this package.

Readings adopted (the pages give no layout):
* a paged cache is a pool of rows [P][D] shared by the batch plus a block
  table [B][max_blocks] of page numbers; row i of sequence b is pool row
  table[b][i // page] * page + i % page;
* a ragged batch gives every sequence its own length t_b: n_b =
  max(0, floor((t_b - W) / s)) compressed entries, min(t_b, W) window rows,
  its own top-k over its own n_b entries, and its own output rotation -t_b.
A ragged, paged step is exactly the per-sequence steps of the uniform path
run one sequence at a time on the rows the tables point to.
"""
from __future__ import annotations

import numpy as np

from .attention import shared_kv_decode
from .compress import n_entries
from .indexer import index_topk


def paged_rows(pool, table, count: int, page: int) -> np.ndarray:
    """The first `count` rows of one sequence: pool [P][D], table [max_blocks]."""
    pool = np.asarray(pool)
    table = np.asarray(table, dtype=np.int64)
    i = np.arange(count)
    return pool[table[i // page] * page + i % page]


def ragged_c4a_step(q, qidx, key_pool, key_tables, comp_pool, comp_tables, win_pool, win_tables, t, page: int,
                    k: int = 512, window: int = 128, stride: int = 4, scale: float = 512 ** -0.5,
                    rope_dim: int = 64, base: float = 10000.0):
    """One c4a layer step of a ragged, paged batch: per sequence b, the top-k
    of its n_b indexer keys, then one softmax over the selected entries and
    its min(t_b, W) window rows, rotated by -t_b.  Returns (idx [B][k],
    counts [B], out [B][H][D])."""
    idx, cnt, out = [], [], []
    for b in range(len(q)):
        n_b = n_entries(int(t[b]), window, stride)
        w_b = min(int(t[b]), window)
        keys = paged_rows(key_pool, key_tables[b], n_b, page)
        sel, c = index_topk(qidx[b], keys, k)
        comp = paged_rows(comp_pool, comp_tables[b], n_b, page)
        win = paged_rows(win_pool, win_tables[b], w_b, page)
        rows = np.concatenate([comp[sel[sel >= 0]], win], axis=0)
        idx.append(sel)
        cnt.append(c)
        out.append(shared_kv_decode(q[b], rows, scale, int(t[b]), rope_dim, base))
    return np.stack(idx), np.array(cnt), np.stack(out)


def ragged_c128a_step(q, comp_pool, comp_tables, win_pool, win_tables, t, page: int, window: int = 128,
                      stride: int = 128, scale: float = 512 ** -0.5, rope_dim: int = 64,
                      base: float = 10000.0) -> np.ndarray:
    """One c128a layer step of a ragged, paged batch: per sequence b, one
    softmax over all its n_b compressed entries and its min(t_b, W) window
    rows, rotated by -t_b ([P1] "c128a": full attention over the compressed
    entries).  Returns out [B][H][D]."""
    out = []
    for b in range(len(q)):
        n_b = n_entries(int(t[b]), window, stride)
        w_b = min(int(t[b]), window)
        rows = np.concatenate([paged_rows(comp_pool, comp_tables[b], n_b, page),
                               paged_rows(win_pool, win_tables[b], w_b, page)], axis=0)
        out.append(shared_kv_decode(q[b], rows, scale, int(t[b]), rope_dim, base))
    return np.stack(out)
