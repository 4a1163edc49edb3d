"""Pins for oracle.indexer: brute force, ties, k >= N, permutation, split/merge."""
import numpy as np
import pytest

from oracle import indexer as I


def _brute(q, keys, k):
    n = len(keys)
    sc = [sum(int(a) * int(b) for a, b in zip(q, row)) for row in keys]
    sel = sorted(sorted(range(n), key=lambda i: (-sc[i], i))[:k])
    return sel + [-1] * (k - len(sel)), sc


@pytest.mark.parametrize("n,k", [(50, 16), (200, 64), (10, 16), (64, 64), (0, 8), (1, 4)])
def test_against_brute_force(n, k):
    rng = np.random.default_rng(n * 100 + k)
    q = rng.integers(-8, 9, 128)
    keys = rng.integers(-2, 3, (n, 128))        # narrow values: many ties
    idx, cnt = I.index_topk(q, keys, k)
    ref, sc = _brute(q, keys, k)
    assert list(idx) == ref
    assert cnt == min(n, k)
    if n:
        assert np.array_equal(I.scores(q, keys), np.array(sc, dtype=np.float64))


def test_ties_go_to_lower_index():
    idx, cnt = I.topk(np.zeros(1000), 512)
    assert list(idx) == list(range(512)) and cnt == 512
    s = np.zeros(20)
    s[[3, 9, 15]] = 5.0
    idx, _ = I.topk(s, 5)
    assert list(idx) == [0, 1, 3, 9, 15]


def test_k_at_least_n_selects_everything():
    idx, cnt = I.topk(np.arange(480, dtype=float)[::-1], 512)
    assert cnt == 480 and list(idx[:480]) == list(range(480)) and np.all(idx[480:] == -1)


def test_permutation_equivariance():
    rng = np.random.default_rng(7)
    s = rng.permutation(5000).astype(float)        # distinct scores
    perm = rng.permutation(5000)
    a, _ = I.topk(s, 512)
    b, _ = I.topk(s[perm], 512)
    assert sorted(perm[b]) == list(a)


def test_split_then_merge_equals_global():
    rng = np.random.default_rng(8)
    s = rng.integers(-300, 300, 32736).astype(float)
    glob, _ = I.topk(s, 512)
    cand = []
    for lo in range(0, len(s), 3000):
        loc, c = I.topk(s[lo:lo + 3000], 512)
        cand.extend(lo + loc[:c])
    cand = np.array(sorted(cand))
    sub, c = I.topk(s[cand], 512)
    assert list(cand[sub[:c]]) == list(glob)


# ------------------------------------------------------------ pool re-index
def _int_data(seed, n, di=128):
    rng = np.random.default_rng(seed)
    return rng.integers(-8, 9, di).astype(np.float64), rng.integers(-8, 9, (n, di)).astype(np.float64)


def test_pool_of_everything_is_the_full_selection():
    q, keys = _int_data(3, 3000)
    full, c1 = I.index_topk(q, keys, 512)
    pooled, c2 = I.index_topk_pool(q, keys, np.arange(3000), 512)
    assert c1 == c2 and np.array_equal(full, pooled)


def test_pool_against_brute_force_and_padding():
    q, keys = _int_data(4, 5000)
    rng = np.random.default_rng(9)
    pool = np.sort(rng.choice(5000, 1500, replace=False))
    padded = np.concatenate([pool, -np.ones(548, dtype=np.int64)])
    got, cnt = I.index_topk_pool(q, keys, padded, 512)
    # brute force: rank every pool entry by (score desc, index asc) with Python tuples
    s = {int(i): float(keys[i] @ q) for i in pool}
    ranked = sorted(pool.tolist(), key=lambda i: (-s[i], i))
    assert cnt == 512
    assert got.tolist() == sorted(ranked[:512])
    # a pool smaller than k: everything, ascending, padded
    small, c = I.index_topk_pool(q, keys, pool[:100], 512)
    assert c == 100 and small[:100].tolist() == pool[:100].tolist() and np.all(small[100:] == -1)


def test_pool_order_and_duplicated_scores():
    """The pool's order does not matter; equal scores go to the lower entry."""
    keys = np.zeros((50, 128))
    keys[[7, 3, 41, 12], 0] = 1.0                  # four equal top scores
    q = np.zeros(128)
    q[0] = 1.0
    got, cnt = I.index_topk_pool(q, keys, np.array([41, 12, 7, 3, 20, 30]), 3)
    assert cnt == 3 and got.tolist() == [3, 7, 12]
