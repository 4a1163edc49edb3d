"""dsv4kv_dense_decode / dsv4kv_sparse_decode (bf16 caches) against the oracle."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import attention as OA
from oracle import formats as OF
from oracle import indexer as OI
from tests._util import assert_close, scaled_max_abs, to_f64

pytestmark = pytest.mark.gpu
SCALE = 512 ** -0.5


def _normal(key, shape):
    import datagen.gpu as G
    return G.normal_bf16_(torch.empty(shape, dtype=torch.bfloat16, device="cuda"), key)


def _rows(key, flat_rows):
    return OF.bf16_bits_to_f64(D.rows_normal_bf16(key, np.asarray(flat_rows), 512))


def _inputs(seed, b, h, rows, win_rows):
    kq, kc, kw = (D.stream_key(seed, t, 0) for t in (D.TID_Q, D.TID_COMP, D.TID_WIN))
    q = _normal(kq, (b, h, 512))
    comp = _normal(kc, (b, max(rows, 1), 512))
    win = _normal(kw, (b, max(win_rows, 1), 512))
    return q, comp, win, (kq, kc, kw)


def _q_host(kq, s, h):
    return _rows(kq, np.arange(s * h, (s + 1) * h))


@pytest.mark.parametrize("b,h,n,window,t", [
    (1, 16, 0, 128, 128),          # window only
    (2, 64, 1, 128, 2048),
    (2, 64, 63, 37, 10000),        # ragged tails, short window
    (2, 64, 64, 0, 5000),          # no window
    (1, 16, 200, 128, 131072),
    (2, 33, 1500, 128, 262144),    # odd head count
    (8, 64, 1023, 128, 131072),    # c128a B=8 t=131072 (full size, every sequence)
    (64, 64, 2047, 128, 262144),   # many tiles per CTA
])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_dense_decode(b, h, n, window, t, out_fp32):
    rows, wrows = n + 3, max(window, 1) + 5
    q, comp, win, (kq, kc, kw) = _inputs(1000 + n + h, b, h, rows, wrows)
    ws = K.new_workspace(K.dense_decode_workspace_bytes(b, h, n, window))
    out = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, window, t, SCALE, out_fp32=out_fp32, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    got = to_f64(out)
    check = range(b) if b <= 8 else (0, b // 2, b - 1)
    for s in check:
        comp_rows = _rows(kc, np.arange(s * rows, s * rows + n))
        win_rows = _rows(kw, np.arange(s * wrows, s * wrows + window))
        ref = OA.dense_decode(_q_host(kq, s, h)[None], comp_rows[None], win_rows[None], t, SCALE)[0]
        assert_close(got[s], ref, what=f"seq {s}")


def test_dense_decode_rescales_when_scores_jump():
    """Later tiles score far higher than the first: the TMEM accumulator rescale path."""
    b, h, n, window, t = 148, 16, 1000, 128, 4096   # one CTA per sequence: every tile in one CTA
    kq, kc, kw = (D.stream_key(9, x, 0) for x in (D.TID_Q, D.TID_COMP, D.TID_WIN))
    q = _normal(kq, (b, h, 512))
    comp = _normal(kc, (b, n, 512))
    win = _normal(kw, (b, window, 512))
    factor = torch.ones(n, device="cuda", dtype=torch.float32)
    factor[:300] = 0.05
    factor[300:700] = 2.0
    factor[700:] = 6.0
    comp = (comp.float() * factor[None, :, None]).to(torch.bfloat16)
    out = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, window, t, SCALE, out_fp32=True)
    got = to_f64(out)
    cbits = comp.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in (0, 77, 147):
        comp_rows = OF.bf16_bits_to_f64(cbits[s])
        win_rows = _rows(kw, np.arange(s * window, (s + 1) * window))
        ref = OA.dense_decode(_q_host(kq, s, h)[None], comp_rows[None], win_rows[None], t, SCALE)[0]
        # rows here are scaled up to 6x, so outputs exceed 1: the bound for scaled inputs
        assert_close(got[s], ref, max_abs=scaled_max_abs(ref), what=f"seq {s}")


def _sorted_choice(rng, n, cnt, k):
    sel = np.sort(rng.choice(n, size=cnt, replace=False)).astype(np.int32)
    return np.concatenate([sel, np.full(k - cnt, -1, np.int32)])


@pytest.mark.parametrize("b,h,n,k,cnt,window,t", [
    (1, 16, 480, 512, 480, 128, 2048),     # tiny c4a: every entry selected, 32 pad slots
    (2, 64, 5000, 512, 512, 128, 131072),
    (2, 64, 5000, 100, 100, 128, 131072),  # short k with a ragged tile
    (3, 64, 70, 512, 40, 0, 600),          # no window
    (32, 64, 32736, 512, 512, 128, 131072),  # c4a B=32 t=131072 (full size)
])
def test_sparse_decode(b, h, n, k, cnt, window, t):
    rng = np.random.default_rng(n + k + b)
    rows, wrows = n, max(window, 1)
    q, comp, win, (kq, kc, kw) = _inputs(3000 + n + k, b, h, rows, wrows)
    idx = np.stack([_sorted_choice(rng, n, cnt, k) for _ in range(b)])
    ws = K.new_workspace(K.sparse_decode_workspace_bytes(b, h, k, window))
    out = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, win), torch.from_numpy(idx).cuda(), n, window, t, SCALE,
                          out_fp32=True, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    got = to_f64(out)
    for s in (range(b) if b <= 4 else (0, 11, b - 1)):
        sel = idx[s][idx[s] >= 0]
        comp_rows = np.zeros((n, 512))
        comp_rows[sel] = _rows(kc, s * rows + sel)
        win_rows = _rows(kw, np.arange(s * wrows, s * wrows + window))
        ref = OA.sparse_decode(_q_host(kq, s, h)[None], comp_rows[None], win_rows[None], idx[s][None], t, SCALE)[0]
        assert_close(got[s], ref, what=f"seq {s}")


def test_sparse_decode_skips_and_flags_bad_indices():
    b, h, n, k, window, t = 1, 16, 300, 64, 128, 5000
    q, comp, win, (kq, kc, kw) = _inputs(55, b, h, n, window)
    idx = np.concatenate([np.arange(0, 60, dtype=np.int32), np.array([n + 5, 299, -1, -1], np.int32)])
    ws = K.new_workspace(K.sparse_decode_workspace_bytes(b, h, k, window))
    out = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, win), torch.from_numpy(idx[None]).cuda(), n, window, t,
                          SCALE, out_fp32=True, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) & K.DEV_BAD_INDEX
    keep = idx[(idx >= 0) & (idx < n)]
    comp_rows = _rows(kc, np.arange(n))
    win_rows = _rows(kw, np.arange(window))
    ref = OA.shared_kv_decode(_q_host(kq, 0, h), np.concatenate([comp_rows[keep], win_rows]), SCALE, t)
    assert_close(to_f64(out)[0], ref)


def test_sparse_equals_dense_when_everything_is_selected():
    b, h, n, window, t = 2, 64, 300, 128, 9000
    q, comp, win, _ = _inputs(66, b, h, n, window)
    idx = torch.arange(n, dtype=torch.int32, device="cuda")[None].repeat(b, 1)
    sp = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, win), idx, n, window, t, SCALE, out_fp32=True)
    de = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, window, t, SCALE, out_fp32=True)
    assert_close(to_f64(sp), to_f64(de), max_abs=1e-5, rel_l2=1e-5)


@pytest.mark.parametrize("max_cluster", ["1", "2", "16"])
@pytest.mark.parametrize("kind,b,n,t", [
    ("dense", 1, 8191, 1048576),   # c128a B=1: 130 tiles, merged in groups, then decode_combine(_wide)
    ("dense", 2, 1500, 262144),    # 26 tiles per sequence
    ("sparse", 1, 262112, 1048576),  # c4a B=1: 10 tiles, empty splits padded into one cluster
    ("sparse", 32, 32736, 131072),   # c4a B=32: 4 splits per sequence
])
def test_split_merge_paths(monkeypatch, max_cluster, kind, b, n, t):
    """The same outputs whether the splits of a sequence are merged inside the
    decode kernel (one thread-block cluster per sequence, or per group of
    splits followed by decode_combine) or only by decode_combine."""
    monkeypatch.setenv("DSV4KV_DECODE_MAX_CLUSTER", max_cluster)
    h, window, k = 64, 128, 512
    rows = n if kind == "sparse" else n + 3
    q, comp, win, (kq, kc, kw) = _inputs(5000 + b + n, b, h, rows, window)
    if kind == "dense":
        out = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, window, t, SCALE, out_fp32=True)
    else:
        rng = np.random.default_rng(b + n)
        idx = np.stack([_sorted_choice(rng, n, k, k) for _ in range(b)])
        out = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, win), torch.from_numpy(idx).cuda(), n, window, t,
                              SCALE, out_fp32=True)
    torch.cuda.synchronize()
    got = to_f64(out)
    for s in ((0,) if b == 1 else (0, b - 1)):
        win_rows = _rows(kw, np.arange(s * window, (s + 1) * window))
        if kind == "dense":
            comp_rows = _rows(kc, np.arange(s * rows, s * rows + n))
            ref = OA.dense_decode(_q_host(kq, s, h)[None], comp_rows[None], win_rows[None], t, SCALE)[0]
        else:
            # only the selected rows, renumbered 0..k-1 (the attention is over the set)
            sel_rows = _rows(kc, s * rows + idx[s])
            ref = OA.sparse_decode(_q_host(kq, s, h)[None], sel_rows[None], win_rows[None],
                                   np.arange(k, dtype=np.int32)[None], t, SCALE)[0]
        assert_close(got[s], ref, what=f"seq {s} (max cluster {max_cluster})")


def test_unaligned_workspace_is_rejected():
    """A workspace that is not 16-byte aligned is refused on the host (its
    16-byte statistics stores would otherwise fault); nothing is launched."""
    q, comp, win, _ = _inputs(3, 2, 64, 300, 128)
    n, t = 300, 300 * 128 + 128
    need = K.dense_decode_workspace_bytes(2, 64, n, 128)
    ws = K.new_workspace(need + 32)[8:8 + need + 16]
    assert ws.data_ptr() % 16 == 8
    with pytest.raises(K.Dsv4kvError) as e:
        K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, 128, t, ws=ws)
    assert e.value.status == 1
    # the same call on an aligned workspace runs
    out = K.dense_decode(q, K.Cache(0, comp), K.Cache(0, win), n, 128, t)
    assert torch.isfinite(out.float()).all()
