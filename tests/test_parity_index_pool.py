"""dsv4kv_index_topk_pool (re-index inside a candidate pool) against the
oracle: bit-exact index sets and counts."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import formats as OF
from oracle import indexer as OI

pytestmark = pytest.mark.gpu


def _keys_bf16(seed, b, n, lo=-8, hi=8):
    import datagen.gpu as G
    kk = D.stream_key(seed, D.TID_KIDX, 0)
    keys = G.int_bf16_(torch.empty(b, n, 128, dtype=torch.bfloat16, device="cuda"), kk, lo, hi)
    return keys, kk


def _q(seed, b):
    import datagen.gpu as G
    kq = D.stream_key(seed, D.TID_QIDX, 0)
    return G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), kq, -8, 8), kq


def _host_q(kq, s):
    return OF.bf16_bits_to_f64(D.rows_int_bf16(kq, np.array([s]), 128)[0])


def _check(idx, cnt, pool, qh, kh, k, s):
    ref, c = OI.index_topk_pool(qh, kh, pool, k)
    assert int(cnt) == c, f"seq {s}: count {int(cnt)} vs {c}"
    assert np.array_equal(idx, ref), f"seq {s}"


@pytest.mark.parametrize("b,n,pool_k,k", [(3, 5000, 2048, 512), (2, 20000, 2048, 512), (2, 3000, 600, 512),
                                          (1, 9000, 8192, 2048), (2, 30000, 5000, 512), (4, 700, 300, 64)])
def test_pool_from_a_full_layer(b, n, pool_k, k):
    """The Full layer's top-pool_k (another query; an ascending random pool when
    pool_k is beyond dsv4kv_index_topk's k) is the pool; this layer's query
    re-ranks it."""
    keys, kk = _keys_bf16(40 + n, b, n)
    q_full, _ = _q(41 + n, b)
    q, kq = _q(42 + n, b)
    cache = K.Cache(0, keys, None, 128)
    if pool_k <= 2048:
        pool, _ = K.index_topk(q_full, cache, n, pool_k)
    else:
        rng = np.random.default_rng(pool_k)
        pool = torch.from_numpy(np.stack([np.sort(rng.choice(n, pool_k, replace=False)) for _ in range(b)])
                                .astype(np.int32)).cuda()
    ws = K.new_workspace(16)
    idx, cnt = K.index_topk_pool(q, cache, n, pool, k, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    idx, cnt, poolh = idx.cpu().numpy(), cnt.cpu().numpy(), pool.cpu().numpy()
    for s in range(b):
        kh = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128))
        _check(idx[s], cnt[s], poolh[s], _host_q(kq, s), kh, k, s)


def test_pool_of_all_entries_equals_index_topk():
    b, n, k = 3, 6000, 512
    keys, _ = _keys_bf16(50, b, n)
    q, _ = _q(51, b)
    cache = K.Cache(0, keys, None, 128)
    pool = torch.arange(n, dtype=torch.int32, device="cuda").repeat(b, 1).contiguous()
    a, ca = K.index_topk_pool(q, cache, n, pool, k)
    r, cr = K.index_topk(q, cache, n, k)
    assert torch.equal(a, r) and torch.equal(ca, cr)


@pytest.mark.parametrize("lo,hi", [(-1, 1), (0, 1), (0, 0)])
def test_pool_heavy_ties(lo, hi):
    """Narrow key values: thousands of equal scores; ties go to the lower entry."""
    b, n, k = 2, 12000, 512
    keys, kk = _keys_bf16(60 + lo + hi, b, n, lo, hi)
    q, kq = _q(61, b)
    rng = np.random.default_rng(3)
    poolh = np.stack([np.sort(rng.choice(n, 5000, replace=False)) for _ in range(b)]).astype(np.int32)
    idx, cnt = K.index_topk_pool(q, K.Cache(0, keys, None, 128), n, torch.from_numpy(poolh).cuda(), k)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for s in range(b):
        kh = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128, lo, hi))
        _check(idx[s], cnt[s], poolh[s], _host_q(kq, s), kh, k, s)


def test_pool_padding_and_small_pools():
    b, n, k = 3, 4000, 512
    keys, kk = _keys_bf16(70, b, n)
    q, kq = _q(71, b)
    rng = np.random.default_rng(4)
    poolh = -np.ones((b, 1024), dtype=np.int32)
    sizes = [1024, 700, 0]                          # full, padded with -1 (more than k), empty
    for s, m in enumerate(sizes):
        poolh[s, :m] = np.sort(rng.choice(n, m, replace=False))
    small = np.full((b, 100), -1, dtype=np.int32)   # fewer than k entries
    small[:, :90] = np.sort(rng.choice(n, 90, replace=False))
    for ph in (poolh, small):
        idx, cnt = K.index_topk_pool(q, K.Cache(0, keys, None, 128), n, torch.from_numpy(ph).cuda(), k)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        for s in range(b):
            kh = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128))
            _check(idx[s], cnt[s], ph[s], _host_q(kq, s), kh, k, s)


def test_pool_fp4_keys():
    import datagen.gpu as G
    b, n, k = 3, 20000, 512
    kf = D.stream_key(8, D.TID_KIDX_FP4, 0)
    codes = torch.empty(b, n, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(b, n, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, kf)
    cache = K.Cache(2, codes, scales, 128)
    q_full, _ = _q(81, b)
    q, kq = _q(82, b)
    pool, _ = K.index_topk(q_full, cache, n, 2048)
    idx, cnt = K.index_topk_pool(q, cache, n, pool, k)
    idx, cnt, poolh = idx.cpu().numpy(), cnt.cpu().numpy(), pool.cpu().numpy()
    for s in range(b):
        hc, hs = D.fp4_index_keys_rows(kf, np.arange(s * n, (s + 1) * n), 128)
        _check(idx[s], cnt[s], poolh[s], _host_q(kq, s), OF.dequant_fp4_rows(hc, hs), k, s)


def test_pool_full_size_sampled():
    """c4a B=32, n=32736: the Full layer's top-2048 as the pool, sampled sequences."""
    b, n, k = 32, 32736, 512
    keys, kk = _keys_bf16(90, b, n)
    q_full, _ = _q(91, b)
    q, kq = _q(92, b)
    cache = K.Cache(0, keys, None, 128)
    pool, _ = K.index_topk(q_full, cache, n, 2048)
    idx, cnt = K.index_topk_pool(q, cache, n, pool, k)
    idx, cnt, poolh = idx.cpu().numpy(), cnt.cpu().numpy(), pool.cpu().numpy()
    for s in (0, 17, 31):
        kh = OF.bf16_bits_to_f64(D.rows_int_bf16(kk, np.arange(s * n, (s + 1) * n), 128))
        _check(idx[s], cnt[s], poolh[s], _host_q(kq, s), kh, k, s)


def test_pool_flags_bad_entries():
    """An entry >= n and a pool out of order are reported in the status word."""
    b, n, k = 1, 1000, 16
    keys, _ = _keys_bf16(95, b, n)
    q, _ = _q(96, b)
    cache = K.Cache(0, keys, None, 128)
    ws = K.new_workspace(16)
    K.index_topk_pool(q, cache, n, torch.tensor([[1, 5, 1000 + 7, 9]], dtype=torch.int32, device="cuda"), k, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) & K.DEV_BAD_INDEX
    ws2 = K.new_workspace(16)
    K.index_topk_pool(q, cache, n, torch.tensor([[9, 5, 7]], dtype=torch.int32, device="cuda"), k, ws=ws2)
    torch.cuda.synchronize()
    assert K.workspace_status(ws2) & K.DEV_BAD_POOL
