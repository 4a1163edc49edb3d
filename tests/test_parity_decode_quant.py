"""Decode over fp8 (E4M3, per-row scale) and fp4 (E2M1, E4M3 scale per 16)
caches, quantised on the GPU by dsv4kv_quantize from seeded N(0,1) states,
against the oracle run on its own quantisation of the same states (the codes
are bit-exact, so both sides attend over identical dequantised rows)."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from datagen import workloads as W
from oracle import attention as OA
from oracle import formats as OF
from tests._util import assert_close, scaled_max_abs, to_f64

pytestmark = pytest.mark.gpu
SCALE = 512 ** -0.5
QUANT = {K.FP8_E4M3_ROW: OF.quantize_fp8_rows, K.FP4_E2M1_G16: OF.quantize_fp4_rows,
         K.FP8_E4M3_ROW_ROPE_BF16: OF.quantize_fp8_rope_rows}
DEQ = {K.FP8_E4M3_ROW: OF.dequant_fp8_rows, K.FP4_E2M1_G16: OF.dequant_fp4_rows,
       K.FP8_E4M3_ROW_ROPE_BF16: OF.dequant_fp8_rope_rows}
FMTS = [K.FP8_E4M3_ROW, K.FP4_E2M1_G16, K.FP8_E4M3_ROW_ROPE_BF16]


def _states(key, b, rows):
    import datagen.gpu as G
    return G.normal_bf16_(torch.empty(b, rows, 512, dtype=torch.bfloat16, device="cuda"), key)


def _host_rows(fmt, key, flat_rows):
    x = OF.bf16_bits_to_f64(D.rows_normal_bf16(key, np.asarray(flat_rows), 512)).astype(np.float32)
    return DEQ[fmt](*QUANT[fmt](x))


def _setup(seed, fmt, b, h, rows, window):
    kq, kc, kw = (D.stream_key(seed, t, fmt) for t in (D.TID_Q, D.TID_STATES, D.TID_WIN))
    import datagen.gpu as G
    q = G.normal_bf16_(torch.empty(b, h, 512, dtype=torch.bfloat16, device="cuda"), kq)
    cc, cs = K.quantize(_states(kc, b, rows), fmt)
    wc, wsc = K.quantize(_states(kw, b, max(window, 1)), fmt)
    return q, K.Cache(fmt, cc, cs), K.Cache(fmt, wc, wsc), (kq, kc, kw)


def _qh(kq, s, h):
    return OF.bf16_bits_to_f64(D.rows_normal_bf16(kq, np.arange(s * h, (s + 1) * h), 512))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("b,h,n,window,t", [
    (1, 16, 0, 128, 128),
    (2, 64, 100, 128, 13000),
    (3, 64, 1023, 37, 131072),
    (64, 64, 2047, 128, 262144),     # quantised c128a, B=64 t=262144 (full size)
])
def test_dense_decode_quantised(fmt, b, h, n, window, t):
    q, comp, win, (kq, kc, kw) = _setup(10 + n, fmt, b, h, max(n, 1), window)
    ws = K.new_workspace(K.dense_decode_workspace_bytes(b, h, n, window))
    out = K.dense_decode(q, comp, win, n, window, t, SCALE, out_fp32=True, ws=ws)
    torch.cuda.synchronize()
    assert K.workspace_status(ws) == 0
    got = to_f64(out)
    rows, wrows = max(n, 1), max(window, 1)
    for s in (range(b) if b <= 3 else (0, 31, b - 1)):
        cr = _host_rows(fmt, kc, np.arange(s * rows, s * rows + n)) if n else np.zeros((0, 512))
        wr = _host_rows(fmt, kw, np.arange(s * wrows, s * wrows + window))
        ref = OA.dense_decode(_qh(kq, s, h)[None], cr[None], wr[None], t, SCALE)[0]
        assert_close(got[s], ref, what=f"fmt {fmt} seq {s}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("b,h,n,k,cnt,t", [
    (2, 64, 3000, 512, 512, 20000),
    (2, 16, 300, 512, 300, 2000),
    (64, 64, 65504, 512, 512, 262144),   # quantised c4a, B=64 t=262144 (full size)
])
def test_sparse_decode_quantised(fmt, b, h, n, k, cnt, t):
    window = 128
    rng = np.random.default_rng(n + fmt)
    q, comp, win, (kq, kc, kw) = _setup(20 + n, fmt, b, h, n, window)
    idx = np.stack([np.concatenate([np.sort(rng.choice(n, cnt, replace=False)), -np.ones(k - cnt)]).astype(np.int32)
                    for _ in range(b)])
    out = K.sparse_decode(q, comp, win, torch.from_numpy(idx).cuda(), n, window, t, SCALE, out_fp32=True)
    got = to_f64(out)
    for s in (range(b) if b <= 2 else (0, b - 1)):
        sel = idx[s][idx[s] >= 0]
        cr = np.zeros((n, 512))
        cr[sel] = _host_rows(fmt, kc, s * n + sel)
        wr = _host_rows(fmt, kw, np.arange(s * window, (s + 1) * window))
        ref = OA.sparse_decode(_qh(kq, s, h)[None], cr[None], wr[None], idx[s][None], t, SCALE)[0]
        assert_close(got[s], ref, what=f"fmt {fmt} seq {s}")


def test_fp8_rows_with_large_scales():
    """Row scales far above 1 (amax ~ 1e4): the weights carry the scale, the
    accumulator stays in range (the m_o / m_l split)."""
    b, h, n, window, t = 2, 64, 500, 128, 5000
    kq, kc, kw = (D.stream_key(77, x, 0) for x in (D.TID_Q, D.TID_STATES, D.TID_WIN))
    import datagen.gpu as G
    q = G.normal_bf16_(torch.empty(b, h, 512, dtype=torch.bfloat16, device="cuda"), kq)
    st = _states(kc, b, n)
    mult = torch.logspace(-2, 4, n, device="cuda")[None, :, None]
    st = (st.float() * mult).to(torch.bfloat16)
    q = (q.float() / 64).to(torch.bfloat16)        # keep the softmax from collapsing onto one row
    cc, cs = K.quantize(st, K.FP8_E4M3_ROW)
    wc, wsc = K.quantize(_states(kw, b, window), K.FP8_E4M3_ROW)
    out = K.dense_decode(q, K.Cache(1, cc, cs), K.Cache(1, wc, wsc), n, window, t, SCALE, out_fp32=True)
    got = to_f64(out)
    qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
    sb = st.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(b):
        cr = OF.dequant_fp8_rows(*OF.quantize_fp8_rows(OF.bf16_bits_to_f64(sb[s]).astype(np.float32)))
        wr = _host_rows(K.FP8_E4M3_ROW, kw, np.arange(s * window, (s + 1) * window))
        ref = OA.dense_decode(OF.bf16_bits_to_f64(qb[s])[None], cr[None], wr[None], t, SCALE)[0]
        assert_close(got[s], ref, max_abs=scaled_max_abs(ref), what=f"seq {s}")


def test_fp8_rope_rows_with_large_rotary_channels():
    """fp8 rows with bf16 rotary channels whose rotary values are 50 times the
    body's: the rotary channels are staged as f16 of value / row scale (here
    up to ~2e4, inside the f16 range), so the output still matches."""
    fmt = K.FP8_E4M3_ROW_ROPE_BF16
    b, h, n, window, t = 2, 64, 700, 128, 9000
    kq, kc, kw = (D.stream_key(91, x, 0) for x in (D.TID_Q, D.TID_STATES, D.TID_WIN))
    import datagen.gpu as G
    q = G.normal_bf16_(torch.empty(b, h, 512, dtype=torch.bfloat16, device="cuda"), kq)
    q = (q.float() / 16).to(torch.bfloat16)        # keep the softmax from collapsing onto one row
    st = _states(kc, b, n).float()
    st[..., 448:] *= 50.0
    st = st.to(torch.bfloat16)
    cc, cs = K.quantize(st, fmt)
    wc, wsc = K.quantize(_states(kw, b, window), fmt)
    out = K.dense_decode(q, K.Cache(fmt, cc, cs), K.Cache(fmt, wc, wsc), n, window, t, SCALE, out_fp32=True)
    got = to_f64(out)
    qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
    sb = st.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(b):
        cr = OF.dequant_fp8_rope_rows(*OF.quantize_fp8_rope_rows(OF.bf16_bits_to_f64(sb[s]).astype(np.float32)))
        wr = _host_rows(fmt, kw, np.arange(s * window, (s + 1) * window))
        ref = OA.dense_decode(OF.bf16_bits_to_f64(qb[s])[None], cr[None], wr[None], t, SCALE)[0]
        # outputs of the rotary channels reach ~50x the usual magnitude: the bound for scaled inputs
        assert_close(got[s], ref, max_abs=scaled_max_abs(ref), what=f"seq {s}")
