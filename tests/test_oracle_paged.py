"""Pins for oracle.paged: an identity block table is the contiguous cache,
shuffled pages with the matching table give the same rows, and a ragged step
with equal lengths is the uniform batched step."""
import numpy as np

from oracle import attention as A
from oracle import compress as C
from oracle import indexer as I
from oracle import paged as P


def test_identity_table_is_the_contiguous_cache():
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((3 * 256, 8))
    table = np.arange(3)
    assert np.array_equal(P.paged_rows(rows, table, 700, 256), rows[:700])


def test_shuffled_pages_with_their_table_give_the_same_rows():
    rng = np.random.default_rng(2)
    page, pages = 64, 10
    rows = rng.standard_normal((page * pages, 4))
    perm = rng.permutation(pages)                  # logical page j is stored at physical page perm[j]
    pool = np.empty_like(rows)
    for j in range(pages):
        pool[perm[j] * page:(perm[j] + 1) * page] = rows[j * page:(j + 1) * page]
    got = P.paged_rows(pool, perm, 600, page)
    # brute force, row by row
    want = np.stack([rows[i] for i in range(600)])
    assert np.array_equal(got, want)


def _setup(rng, b, t, page, d=512, di=128, heads=4):
    n = [C.n_entries(tb, 128, 4) for tb in t]
    npages = [(max(x, 1) + page - 1) // page for x in n]
    wpages = [(min(tb, 128) + page - 1) // page for tb in t]
    kpool = rng.integers(-8, 9, (sum(npages) * page, di)).astype(np.float64)
    cpool = rng.standard_normal((sum(npages) * page, d))
    wpool = rng.standard_normal((sum(wpages) * page, d))
    kt, wt, o1, o2 = [], [], 0, 0
    for b_ in range(b):
        kt.append(np.arange(o1, o1 + npages[b_]))
        wt.append(np.arange(o2, o2 + wpages[b_]))
        o1 += npages[b_]
        o2 += wpages[b_]
    q = rng.standard_normal((b, heads, d))
    qi = rng.integers(-8, 9, (b, di)).astype(np.float64)
    return q, qi, kpool, kt, cpool, kt, wpool, wt


def test_equal_lengths_give_the_uniform_batched_step():
    rng = np.random.default_rng(3)
    b, t, page = 2, 4224, 64                          # 1024 entries each
    q, qi, kp, kt, cp, ct, wp, wt = _setup(rng, b, [t, t], page)
    idx, cnt, out = P.ragged_c4a_step(q, qi, kp, kt, cp, ct, wp, wt, [t, t], page)
    n = C.n_entries(t, 128, 4)
    for s in range(b):
        keys = P.paged_rows(kp, kt[s], n, page)
        ref_idx, ref_c = I.index_topk(qi[s], keys, 512)
        assert cnt[s] == ref_c and np.array_equal(idx[s], ref_idx)
    comp = np.stack([P.paged_rows(cp, ct[s], n, page) for s in range(b)])
    win = np.stack([P.paged_rows(wp, wt[s], 128, page) for s in range(b)])
    ref = A.sparse_decode(q, comp, win, idx, t, 512 ** -0.5)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


def test_ragged_lengths_are_independent_sequences():
    """A sequence's result does not depend on the other sequences' lengths."""
    rng = np.random.default_rng(4)
    t = [4224, 700, 90]                               # 1024, 143 and 0 entries (the last: window only, 90 rows)
    q, qi, kp, kt, cp, ct, wp, wt = _setup(rng, 3, t, 64)
    idx, cnt, out = P.ragged_c4a_step(q, qi, kp, kt, cp, ct, wp, wt, t, 64)
    assert list(cnt) == [512, 143, 0] and np.all(idx[2] == -1)
    for s in range(3):
        one = P.ragged_c4a_step(q[s:s + 1], qi[s:s + 1], kp, kt[s:s + 1], cp, ct[s:s + 1], wp, wt[s:s + 1],
                                t[s:s + 1], 64)
        assert np.array_equal(one[0][0], idx[s]) and np.allclose(one[2][0], out[s], rtol=0, atol=0)
    # window-only sequence: textbook softmax attention over its 90 window rows
    win = P.paged_rows(wp, wt[2], 90, 64)
    ref = A.shared_kv_decode(q[2], win, 512 ** -0.5, 90)
    assert np.allclose(out[2], ref, rtol=0, atol=1e-12)


def test_ragged_c128a_with_equal_lengths_is_the_uniform_dense_step():
    rng = np.random.default_rng(5)
    b, t, page = 2, 128 * 40 + 128, 64               # 40 entries each
    n = C.n_entries(t, 128, 128)
    cpool = rng.standard_normal((b * page, 512))
    wpool = rng.standard_normal((2 * b * page, 512))
    ct = [np.array([1]), np.array([0])]               # sequence 0 in page 1, sequence 1 in page 0
    wt = [np.array([3, 2]), np.array([0, 1])]
    q = rng.standard_normal((b, 4, 512))
    out = P.ragged_c128a_step(q, cpool, ct, wpool, wt, [t, t], page)
    comp = np.stack([cpool[page:page + n], cpool[:n]])
    win = np.stack([np.concatenate([wpool[3 * page:4 * page], wpool[2 * page:3 * page]])[:128],
                    wpool[:2 * page][:128]])
    ref = A.dense_decode(q, comp, win, t, 512 ** -0.5)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


def test_ragged_c128a_short_sequences_are_window_only_attention():
    """t_b < W: no compressed entries, t_b window rows, textbook softmax attention."""
    rng = np.random.default_rng(6)
    wpool = rng.standard_normal((3 * 64, 512))
    q = rng.standard_normal((2, 4, 512))
    t = [100, 37]
    out = P.ragged_c128a_step(q, np.zeros((64, 512)), [np.array([0]), np.array([0])], wpool,
                              [np.array([2, 0]), np.array([1])], t, 64)
    for s, (tb, rows) in enumerate([(100, np.concatenate([wpool[128:192], wpool[:64]])[:100]),
                                    (37, wpool[64:101])]):
        sc = q[s] @ rows.T * 512 ** -0.5
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        o = (p / p.sum(axis=1, keepdims=True)) @ rows
        # inverse rotation by -t_b of the last 64 channels (interleaved pairs), written out
        ang = -tb * 10000.0 ** (-np.arange(32) / 32.0)
        x, y = o[:, 448::2].copy(), o[:, 449::2].copy()
        o[:, 448::2] = x * np.cos(ang) - y * np.sin(ang)
        o[:, 449::2] = x * np.sin(ang) + y * np.cos(ang)
        assert np.allclose(out[s], o, rtol=0, atol=1e-12)
