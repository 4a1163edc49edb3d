"""Paged caches of ragged batches (dsv4kv_index_topk_paged,
dsv4kv_sparse_decode_paged, dsv4kv_dense_decode_paged) against the oracle's
ragged, paged steps ([P1] hybrid KV cache manager paragraph: the caches live
in blocks of a shared block pool; every sequence has its own length).

Pages are assigned to sequences in a shuffled order; table entries a sequence
does not use are -1, so a read past a sequence's last row would flag
DEV_BAD_PAGE (every call here must leave its status word at 0).  Lengths mix
a long sequence, medium ones, one with fewer entries than k, one with a
single entry and one shorter than the window."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import formats as OF
from oracle import paged as OP
from tests._util import assert_close, to_f64

pytestmark = pytest.mark.gpu
W = 128


def _tables(rng, counts, page, spare=3):
    """Shuffled page assignment: (table int32 [B][stride], pool pages)."""
    need = [(c + page - 1) // page for c in counts]
    total = sum(need) + spare
    perm = rng.permutation(total).astype(np.int32)
    stride = max(1, max(need))
    table = np.full((len(counts), stride), -1, dtype=np.int32)
    o = 0
    for b, m in enumerate(need):
        table[b, :m] = perm[o:o + m]
        o += m
    return table, total


def _normal_pool(key, rows, d=512):
    import datagen.gpu as G
    dev = G.normal_bf16_(torch.empty(rows, d, dtype=torch.bfloat16, device="cuda"), key)
    host = OF.bf16_bits_to_f64(D.normal_bf16(key, rows * d).reshape(rows, d))
    return dev, host


def _key_pool(key, rows, fmt):
    import datagen.gpu as G
    if fmt == K.BF16:
        dev = G.int_bf16_(torch.empty(rows, 128, dtype=torch.bfloat16, device="cuda"), key)
        return (dev, None), OF.bf16_bits_to_f64(D.int_bf16(key, rows * 128).reshape(rows, 128))
    codes = torch.empty(rows, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, 8, dtype=torch.uint8, device="cuda")
    G.fp4_index_keys_(codes, scales, key)
    hc, hs = D.fp4_index_keys_rows(key, np.arange(rows), 128)
    return (codes, scales), OF.dequant_fp4_rows(hc, hs)


QUANT = {K.FP8_E4M3_ROW: (OF.quantize_fp8_rows, OF.dequant_fp8_rows),
         K.FP4_E2M1_G16: (OF.quantize_fp4_rows, OF.dequant_fp4_rows)}


def _main_pool(key, rows, fmt):
    """(codes, scales) of a main-cache pool and its dequantised rows on the host."""
    dev, host = _normal_pool(key, rows)
    if fmt == K.BF16:
        return (dev, None), host
    codes, scales = K.quantize(dev, fmt)
    q, dq = QUANT[fmt]
    return (codes, scales), dq(*q(host.astype(np.float32)))


def _setup(seed, t, page, main_fmt=K.BF16, key_fmt=K.BF16, stride=4, heads=64, with_keys=True):
    rng = np.random.default_rng(seed)
    n = [max(0, (tb - W) // stride) for tb in t]
    w = [min(tb, W) for tb in t]
    ct, cpages = _tables(rng, n, page)
    wt, wpages = _tables(rng, w, page)
    kc = D.stream_key(seed, D.TID_COMP)
    (cc, cs), c_host = _main_pool(kc, cpages * page, main_fmt)
    (wc, ws_), w_host = _main_pool(D.stream_key(seed, D.TID_WIN), wpages * page, main_fmt)
    import datagen.gpu as G
    b = len(t)
    q = G.normal_bf16_(torch.empty(b, heads, 512, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_Q))
    q_host = OF.bf16_bits_to_f64(D.normal_bf16(D.stream_key(seed, D.TID_Q), b * heads * 512).reshape(b, heads, 512))
    setup = {
        "t": t, "n": n, "page": page, "q": q, "q_host": q_host,
        "comp": K.PagedCache(main_fmt, cc, torch.from_numpy(ct).cuda(), page, cs), "ct": ct, "c_host": c_host,
        "win": K.PagedCache(main_fmt, wc, torch.from_numpy(wt).cuda(), page, ws_), "wt": wt, "w_host": w_host,
        "t_seq": torch.tensor(t, dtype=torch.int64, device="cuda"),
    }
    if with_keys:
        kt, kpages = _tables(rng, n, page)
        kk = D.stream_key(seed, D.TID_KIDX if key_fmt == K.BF16 else D.TID_KIDX_FP4)
        (kcodes, kscales), k_host = _key_pool(kk, kpages * page, key_fmt)
        qidx = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_QIDX))
        setup.update(keys=K.PagedCache(key_fmt, kcodes, torch.from_numpy(kt).cuda(), page, kscales, dim=128), kt=kt,
                     k_host=k_host, qidx=qidx,
                     qidx_host=OF.bf16_bits_to_f64(D.int_bf16(D.stream_key(seed, D.TID_QIDX), b * 128).reshape(b, 128)))
    return setup


C4A_T = [65536, 20000, 2100, 700, 90, 132]   # n = 16352, 4968, 493 (< k), 143, 0 (window only), 1


@pytest.mark.parametrize("page,main_fmt,key_fmt", [(64, K.BF16, K.BF16), (256, K.BF16, K.BF16),
                                                   (64, K.FP8_E4M3_ROW, K.FP4_E2M1_G16),
                                                   (256, K.FP4_E2M1_G16, K.BF16)])
def test_ragged_paged_c4a_step(page, main_fmt, key_fmt):
    S = _setup(11 + page + main_fmt, C4A_T, page, main_fmt, key_fmt)
    t_max = max(C4A_T)
    ws_i = K.new_workspace(K.lib().dsv4kv_index_topk_paged_workspace_bytes(len(C4A_T), t_max, W, 4, 512))
    ws_d = K.new_workspace(K.lib().dsv4kv_sparse_decode_paged_workspace_bytes(len(C4A_T), 64, 512, 512, W))
    idx, cnt = K.index_topk_paged(S["qidx"], S["keys"], S["t_seq"], t_max, 512, ws=ws_i)
    out = K.sparse_decode_paged(S["q"], S["comp"], S["win"], idx, S["t_seq"], t_max, out_fp32=True, ws=ws_d)
    torch.cuda.synchronize()
    assert K.workspace_status(ws_i) == 0 and K.workspace_status(ws_d) == 0
    ref_idx, ref_cnt, ref = OP.ragged_c4a_step(S["q_host"], S["qidx_host"], S["k_host"], S["kt"], S["c_host"],
                                               S["ct"], S["w_host"], S["wt"], C4A_T, page)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    got = to_f64(out)
    for s in range(len(C4A_T)):
        assert_close(got[s], ref[s], what=f"seq {s} (t = {C4A_T[s]})")


C128A_T = [262144, 131072, 5000, 300, 100, 256]   # n = 2047, 1023, 38, 1, 0, 1


@pytest.mark.parametrize("page", [64, 128])
@pytest.mark.parametrize("main_fmt", [K.BF16, K.FP8_E4M3_ROW])
def test_ragged_paged_c128a_step(page, main_fmt):
    S = _setup(21 + page + main_fmt, C128A_T, page, main_fmt, stride=128, with_keys=False)
    t_max = max(C128A_T)
    ws = K.new_workspace(K.lib().dsv4kv_dense_decode_paged_workspace_bytes(len(C128A_T), 64, 512, t_max, W, 128))
    out = K.dense_decode_paged(S["q"], S["comp"], S["win"], S["t_seq"], t_max, out_fp32=True, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    ref = OP.ragged_c128a_step(S["q_host"], S["c_host"], S["ct"], S["w_host"], S["wt"], C128A_T, page)
    got = to_f64(out)
    for s in range(len(C128A_T)):
        assert_close(got[s], ref[s], what=f"seq {s} (t = {C128A_T[s]})")


def test_identity_pages_and_equal_lengths_are_the_dense_layout_calls():
    """Pages laid out in order with one length for all: the paged calls give
    exactly (bit for bit) what the dense-layout calls give on the same memory."""
    import datagen.gpu as G
    b, t, page = 4, 131072, 64
    n = (t - W) // 4
    rows = (n + page - 1) // page * page          # per-sequence capacity: whole pages
    keys = G.int_bf16_(torch.empty(b, rows, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(5, D.TID_KIDX))
    comp = G.normal_bf16_(torch.empty(b, rows, 512, dtype=torch.bfloat16, device="cuda"), D.stream_key(5, D.TID_COMP))
    win = G.normal_bf16_(torch.empty(b, W, 512, dtype=torch.bfloat16, device="cuda"), D.stream_key(5, D.TID_WIN))
    q = G.normal_bf16_(torch.empty(b, 64, 512, dtype=torch.bfloat16, device="cuda"), D.stream_key(5, D.TID_Q))
    qidx = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), D.stream_key(5, D.TID_QIDX))
    per = rows // page
    ctab = (torch.arange(b, dtype=torch.int32)[:, None] * per + torch.arange(per, dtype=torch.int32)[None]).cuda()
    wtab = (torch.arange(b, dtype=torch.int32)[:, None] * 2 + torch.arange(2, dtype=torch.int32)[None]).cuda()
    t_seq = torch.full((b,), t, dtype=torch.int64, device="cuda")
    idx_d, cnt_d = K.index_topk(qidx, K.Cache(0, keys, None, 128), n, 512)
    out_d = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, win), idx_d, n, W, t, out_fp32=True)
    idx_p, cnt_p = K.index_topk_paged(qidx, K.PagedCache(0, keys.view(-1, 128), ctab, page, dim=128), t_seq, t, 512)
    out_p = K.sparse_decode_paged(q, K.PagedCache(0, comp.view(-1, 512), ctab, page),
                                  K.PagedCache(0, win.view(-1, 512), wtab, page), idx_p, t_seq, t, out_fp32=True)
    dense_d = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, W, t, out_fp32=True)
    dense_p = K.dense_decode_paged(q, K.PagedCache(0, comp.view(-1, 512), ctab, page),
                                   K.PagedCache(0, win.view(-1, 512), wtab, page), t_seq, t, stride=4, out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(idx_p, idx_d) and torch.equal(cnt_p, cnt_d)
    assert torch.equal(out_p, out_d)
    assert torch.equal(dense_p, dense_d)


def test_bad_pages_and_lengths_are_flagged_not_faulted():
    S = _setup(31, [40000, 3000], 64)
    t_max = 40000
    keys = S["keys"]
    bad_tab = keys.table.clone()
    bad_tab[0, 3] = keys.pool_pages + 7            # a used page of sequence 0 points outside the pool
    keys_bad = K.PagedCache(keys.fmt, keys.codes, bad_tab, keys.page_rows, keys.scales, dim=128)
    ws_i = K.new_workspace(K.lib().dsv4kv_index_topk_paged_workspace_bytes(2, t_max, W, 4, 512))
    idx, cnt = K.index_topk_paged(S["qidx"], keys_bad, S["t_seq"], t_max, 512, ws=ws_i)
    comp = S["comp"]
    ctab = comp.table.clone()
    ctab[1, 0] = -5
    ws_d = K.new_workspace(K.lib().dsv4kv_sparse_decode_paged_workspace_bytes(2, 64, 512, 512, W))
    out = K.sparse_decode_paged(S["q"], K.PagedCache(comp.fmt, comp.codes, ctab, comp.page_rows), S["win"], idx,
                                S["t_seq"], t_max, out_fp32=True, ws=ws_d)
    long_t = torch.tensor([t_max + 1000, -3], dtype=torch.int64, device="cuda")   # clamped to t_max and 0
    ws_l = K.new_workspace(K.lib().dsv4kv_sparse_decode_paged_workspace_bytes(2, 64, 512, 512, W))
    out_l = K.sparse_decode_paged(S["q"], S["comp"], S["win"], idx, long_t, t_max, out_fp32=True, ws=ws_l)
    torch.cuda.synchronize()
    assert K.workspace_status(ws_i) & K.DEV_BAD_PAGE
    assert K.workspace_status(ws_d) & K.DEV_BAD_PAGE
    assert K.workspace_status(ws_l) & K.DEV_BAD_LENGTH
    assert torch.isfinite(out).all() and torch.isfinite(out_l).all()
    assert (cnt.cpu() == torch.tensor([512, 512], dtype=torch.int32)).all()
