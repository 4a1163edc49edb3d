"""Pins for oracle.attention.

Independent references: torch's scaled_dot_product_attention in float64 (a
library routine) for the window-only and all-selected cases, the single-row
closed form, and the invariants the method fixes (k >= N makes c4a equal
dense; shared K/V equals separate K/V with V := K; row permutation).
"""
import numpy as np
import torch

from oracle import attention as A
from oracle import indexer as I
from oracle import rope as R


def _sdpa(q, rows, scale):
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64))[None]
    kt = torch.from_numpy(np.asarray(rows, dtype=np.float64))[None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, kt.clone(), scale=scale)[0].numpy()


def test_window_only_is_textbook_attention():
    rng = np.random.default_rng(0)
    q = rng.normal(size=(1, 16, 512))
    win = rng.normal(size=(1, 128, 512))
    comp = np.zeros((1, 0, 512))
    t = 128
    out = A.dense_decode(q, comp, win, t, 1 / np.sqrt(512))
    ref = R.rope(_sdpa(q[0], win[0], 1 / np.sqrt(512)), -t)
    assert np.allclose(out[0], ref, rtol=1e-12, atol=1e-12)
    # undoing the output rotation gives plain attention
    assert np.allclose(R.rope(out[0], t), _sdpa(q[0], win[0], 1 / np.sqrt(512)), atol=1e-12)


def test_all_selected_is_textbook_attention_and_equals_dense():
    rng = np.random.default_rng(1)
    b, n, h = 2, 100, 8
    q = rng.normal(size=(b, h, 512))
    comp = rng.normal(size=(b, n, 512))
    win = rng.normal(size=(b, 128, 512))
    idx = np.stack([I.topk(rng.normal(size=n), 512)[0] for _ in range(b)])     # k >= N
    t = 2048
    sp = A.sparse_decode(q, comp, win, idx, t, 0.05)
    de = A.dense_decode(q, comp, win, t, 0.05)
    assert np.allclose(sp, de, atol=1e-13)
    for i in range(b):
        rows = np.concatenate([comp[i], win[i]])
        assert np.allclose(sp[i], R.rope(_sdpa(q[i], rows, 0.05), -t), atol=1e-12)


def test_sparse_reads_only_selected_rows():
    rng = np.random.default_rng(2)
    n = 300
    q = rng.normal(size=(1, 4, 512))
    comp = rng.normal(size=(1, n, 512))
    win = rng.normal(size=(1, 128, 512))
    idx, c = I.topk(rng.normal(size=n), 64)
    out = A.sparse_decode(q, comp, win, idx[None], 4000, 0.1)
    rows = np.concatenate([comp[0][idx[:c]], win[0]])
    assert np.allclose(out[0], R.rope(_sdpa(q[0], rows, 0.1), -4000), atol=1e-12)
    comp2 = comp.copy()
    unused = np.setdiff1d(np.arange(n), idx[:c])
    comp2[0, unused] = 1e3                         # unread rows do not matter
    assert np.array_equal(A.sparse_decode(q, comp2, win, idx[None], 4000, 0.1), out)


def test_single_row_closed_form():
    rng = np.random.default_rng(3)
    q = rng.normal(size=(3, 512))
    row = rng.normal(size=(1, 512))
    out = A.shared_kv_decode(q, row, 0.3, 777)
    assert np.allclose(out, np.repeat(R.rope(row, -777), 3, axis=0), atol=1e-13)


def test_shared_equals_separate_with_v_equal_k_and_permutation():
    rng = np.random.default_rng(4)
    q = rng.normal(size=(8, 512))
    rows = rng.normal(size=(200, 512))
    shared = A.shared_kv_decode(q, rows, 0.04, 0)
    sep = A.attend(q, rows, rows.copy(), 0.04)
    assert np.allclose(shared, sep, atol=1e-14)
    perm = rng.permutation(200)
    assert np.allclose(A.shared_kv_decode(q, rows[perm], 0.04, 0), shared, atol=1e-13)
    # separate values differ: the shared path really uses the keys as values
    other = A.attend(q, rows, rng.normal(size=(200, 512)), 0.04)
    assert not np.allclose(other, shared)


def test_softmax_is_over_the_union():
    """Doubling the window rows' logits changes the comp rows' weights (one softmax)."""
    rng = np.random.default_rng(5)
    q = rng.normal(size=(1, 1, 512))
    comp = rng.normal(size=(1, 10, 512))
    win = rng.normal(size=(1, 5, 512))
    out = A.dense_decode(q, comp, win, 0, 1.0)
    rows = np.concatenate([comp[0], win[0]])
    s = rows @ q[0, 0]
    p = np.exp(s - s.max()); p /= p.sum()
    assert np.allclose(out[0, 0], p @ rows, atol=1e-12)
