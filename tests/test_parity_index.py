"""dsv4kv_index_topk against the oracle: bit-exact index sets and counts."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from datagen import workloads as W
from oracle import formats as OF
from oracle import indexer as OI

pytestmark = pytest.mark.gpu


def _bf16_keys(seed, b, n, lo=-8, hi=8, rows=None):
    import datagen.gpu as G
    rows = rows or n
    kk = D.stream_key(seed, D.TID_KIDX, 0)
    kq = D.stream_key(seed, D.TID_QIDX, 0)
    keys = G.int_bf16_(torch.empty(b, rows, 128, dtype=torch.bfloat16, device="cuda"), kk, lo, hi)
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), kq, -8, 8)
    return q, keys, kk, kq


@pytest.mark.parametrize("b,n,rows,k", [
    (1, 480, 480, 512),        # n < k: everything selected
    (2, 512, 600, 512),        # n == k
    (2, 513, 513, 512),
    (3, 5000, 5003, 512),      # ragged
    (2, 32736, 32736, 512),
    (1, 70000, 70000, 64),
    (2, 9000, 9000, 1),
    (2, 9000, 9000, 2048),
    (150, 1000, 1003, 512),    # many short sequences: a CTA's keys span several sequences
])
def test_index_topk_bf16_small(b, n, rows, k):
    q, keys, kk, kq = _bf16_keys(100 + n + k, b, n, rows=rows)
    ws = K.new_workspace(K.index_topk_workspace_bytes(b, n, k))
    for _ in range(2):   # the workspace is left reusable
        idx, cnt = K.index_topk(q, K.Cache(0, keys, None, 128), n, k, ws=ws)
        torch.cuda.synchronize()
        assert K.workspace_status(ws) == 0
        idx = idx.cpu().numpy()
        cnt = cnt.cpu().numpy()
        for s in range(b):
            kr = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * rows, s * rows + n), 128))
            qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
            ref, c = OI.index_topk(qr, kr, k)
            assert cnt[s] == c
            assert np.array_equal(idx[s], ref), f"seq {s}"


@pytest.mark.parametrize("lo,hi,n", [(-1, 1, 20000), (0, 0, 10000), (0, 1, 50000)])
def test_index_topk_heavy_ties(lo, hi, n):
    """Narrow key values: thousands of equal scores at the cut (the general path)."""
    b, k = 2, 512
    q, keys, kk, kq = _bf16_keys(7 + n, b, n, lo, hi)
    idx, cnt = K.index_topk(q, K.Cache(0, keys, None, 128), n, k)
    idx = idx.cpu().numpy()
    for s in range(b):
        kr = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128, lo, hi))
        qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
        ref, _ = OI.index_topk(qr, kr, k)
        assert np.array_equal(idx[s], ref)


@pytest.mark.parametrize("b,n,rows", [
    (3, 20000, 20000),
    (1, 5001, 5001),      # an odd number of rows: the last key's scale row is not in a 16-byte unit of its own
    (3, 4999, 5003),      # sequences start on odd rows
    (17, 3001, 3001),     # batch >= 16: the shared tail queue, odd total
    (150, 1000, 1001),    # many short sequences per CTA
])
def test_index_topk_fp4_keys(b, n, rows):
    import datagen.gpu as G
    k = 512
    kf = D.stream_key(5 + n, D.TID_KIDX_FP4, 0)
    kq = D.stream_key(5 + n, D.TID_QIDX, 0)
    codes = torch.empty(b, rows, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(b, rows, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, kf)
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), kq)
    ws = K.new_workspace(K.index_topk_workspace_bytes(b, n, k))
    idx, cnt = K.index_topk(q, K.Cache(2, codes, scales, 128), n, k, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    idx = idx.cpu().numpy()
    for s in (range(b) if b <= 17 else (0, 77, b - 1)):
        hc, hs = D.fp4_index_keys_rows(kf, np.arange(s * rows, s * rows + n), 128)
        kr = OF.dequant_fp4_rows(hc, hs)
        qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
        ref, c = OI.index_topk(qr, kr, k)
        assert np.array_equal(idx[s], ref), f"seq {s}"


@pytest.mark.parametrize("wl,sample", [(W.C4A_B32, [0, 13, 31]), (W.STACK_C4A, [0])])
def test_index_topk_full_size_sampled(wl, sample):
    b, n, k = wl.batch, wl.n, wl.k
    q, keys, kk, kq = _bf16_keys(2024, b, n)
    idx, cnt = K.index_topk(q, K.Cache(0, keys, None, 128), n, k)
    idx = idx.cpu().numpy()
    for s in sample:
        kr = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128))
        qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
        ref, _ = OI.index_topk(qr, kr, k)
        assert np.array_equal(idx[s], ref), f"seq {s}"
    # every sequence: valid, ascending, unique
    assert np.all(np.diff(idx, axis=1) > 0) and idx.min() >= 0 and idx.max() < n


def test_index_topk_full_size_fp4_sampled():
    import datagen.gpu as G
    wl = W.Q_C4A_FP8
    b, n, k = wl.batch, wl.n, wl.k
    kf = D.stream_key(77, D.TID_KIDX_FP4, 0)
    kq = D.stream_key(77, D.TID_QIDX, 0)
    codes = torch.empty(b, n, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(b, n, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, kf)
    q = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), kq)
    idx, _ = K.index_topk(q, K.Cache(2, codes, scales, 128), n, k)
    idx = idx.cpu().numpy()
    for s in (0, 63):
        hc, hs = D.fp4_index_keys_rows(kf, np.arange(s * n, (s + 1) * n), 128)
        qr = OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])
        ref, _ = OI.index_topk(qr, OF.dequant_fp4_rows(hc, hs), k)
        assert np.array_equal(idx[s], ref)


@pytest.mark.parametrize("b,n,k", [(2, 300, 512), (3, 5000, 512), (32, 32736, 512)])
def test_index_score_then_select_equals_index_topk(b, n, k):
    """The two-step form (dsv4kv_index_score; dsv4kv_index_select) on one
    workspace gives index_topk's result, call after call."""
    q, keys, kk, kq = _bf16_keys(300 + n, b, n)
    cache = K.Cache(0, keys, None, 128)
    ref_idx, ref_cnt = K.index_topk(q, cache, n, k)
    ws = K.new_workspace(K.index_topk_workspace_bytes(b, n, k))
    idx = torch.empty(b, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(b, dtype=torch.int32, device="cuda")
    for _ in range(3):
        idx.fill_(-7)
        K.index_score(q, cache, n, k, ws)
        K.index_select(b, n, k, idx, cnt, ws)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)
        assert K.workspace_status(ws) == 0


@pytest.mark.parametrize("n_hot", [60, 1000])
def test_index_topk_hot_entries_with_exact_ties(n_hot):
    """n_hot evenly spaced entries score far above everything else, all with
    exactly the same score: with 60 of them the rest of the selection comes
    from the bulk of the scores; with 1000 the top-k is 512 of the equal hot
    entries, which the tie rule resolves to the lowest indices."""
    b, n, k = 2, 40000, 512
    q, keys, kk, kq = _bf16_keys(4242 + n_hot, b, n, -1, 1)
    qsign = torch.where(q.float() >= 0, 1.0, -1.0).to(torch.bfloat16)
    hot = [(j * n) // 1024 for j in range(n_hot)]
    assert n_hot <= 1024 and max(hot) < n
    pos = torch.tensor(hot, device="cuda")
    for s in range(b):
        keys[s, pos] = 8 * qsign[s]
    idx, cnt = K.index_topk(q, K.Cache(0, keys, None, 128), n, k)
    qh = q.float().cpu().double().numpy()
    kh = keys.float().cpu().double().numpy()
    for s in range(b):
        ref_idx, ref_cnt = OI.index_topk(qh[s], kh[s], k)
        assert np.array_equal(idx[s].cpu().numpy(), ref_idx), f"seq {s}"
        assert int(cnt[s]) == ref_cnt
