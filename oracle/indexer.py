"""Lightning-indexer scores and top-k selection (oracle side).

[P1] "c4a (the milder scheme)": DeepSeek Sparse Attention picks the top-k
compressed entries per query, default k = 512; the indexer scores which
entries to read and holds 128 values per entry ("To judge the saving" and the
indexer paragraph).  [P2] Step 5: a learned indexer scores compressed blocks
and the query reads only the selected ones.

Reading adopted: a single 128-dim dot score_i = sum_d q[d] * key_i[d] (no
activation, no head weights); the selected set is the first min(k, N) entries
under the order (score descending, index ascending), i.e. ties go to the lower
index; it is returned in ascending index order, padded with -1 to k.
"""
from __future__ import annotations

import numpy as np


def scores(q, keys) -> np.ndarray:
    """q [Di], keys [N][Di] -> float64 scores [N]."""
    return np.asarray(keys, dtype=np.float64) @ np.asarray(q, dtype=np.float64)


def topk(score, k: int) -> tuple[np.ndarray, int]:
    """-> (idx int32 [k] ascending, -1 padded; count)."""
    score = np.asarray(score, dtype=np.float64)
    n = score.shape[0]
    order = np.lexsort((np.arange(n), -score))     # last key is primary
    cnt = min(k, n)
    sel = np.sort(order[:cnt])
    out = np.full(k, -1, dtype=np.int32)
    out[:cnt] = sel
    return out, cnt


def index_topk(q, keys, k: int) -> tuple[np.ndarray, int]:
    return topk(scores(q, keys), k)


def index_topk_pool(q, keys, pool, k: int) -> tuple[np.ndarray, int]:
    """Re-index inside a candidate pool ([P3] CSA2: "Reindex" layers keep their
    indexing inside the candidate pool built by the first layer in Full mode;
    layers share the indexer keys).  pool: entry indices (negative = no
    entry).  Among the pool entries, the first min(k, |pool|) under (score
    descending, entry index ascending), returned in ascending entry order,
    padded with -1 to k.  Reading: the pool is a set of entry indices; its
    size is the caller's choice (the pages give none)."""
    pool = np.asarray(pool, dtype=np.int64)
    ent = pool[pool >= 0]
    s = scores(q, np.asarray(keys)[ent])
    order = np.lexsort((ent, -s))                   # score desc, then entry index asc
    cnt = min(k, ent.shape[0])
    sel = np.sort(ent[order[:cnt]])
    out = np.full(k, -1, dtype=np.int32)
    out[:cnt] = sel
    return out, cnt
