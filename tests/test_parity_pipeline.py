"""The tiny c4a layer end to end: raw states -> compress -> index/top-k ->
sparse decode, every step on the GPU, against the oracle run from the same
raw states (t = 2048, 480 entries, 16 heads, window 128)."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from datagen import workloads as W
from oracle import attention as OA
from oracle import compress as OC
from oracle import formats as OF
from oracle import indexer as OI
from oracle import rope as OR
from tests._util import assert_close, to_f64

pytestmark = pytest.mark.gpu


def test_tiny_c4a_layer_end_to_end():
    import datagen.gpu as G
    wl = W.TINY_C4A
    b, t, h, win, k = wl.batch, wl.t, wl.heads, wl.window, wl.k
    keys = W.keys_for(1, 0)
    raw = G.normal_bf16_(torch.empty(b, t, 512, dtype=torch.bfloat16, device="cuda"), keys["raw"])
    w = D.compress_weights(1, 0, 8, 512)
    comp = K.compress(raw, torch.from_numpy(w).cuda(), 4, win)                      # [1][480][512] bf16
    one = torch.ones(1, 512, dtype=torch.float32, device="cuda")
    window = K.compress(raw[:, t - win:].contiguous(), one, 1, 0, pos0=t - win)      # rotated window rows
    n = comp.shape[1]
    assert n == 480
    kidx = G.int_bf16_(torch.empty(b, n, 128, dtype=torch.bfloat16, device="cuda"), keys["kidx"])
    qidx = G.int_bf16_(torch.empty(b, 128, dtype=torch.bfloat16, device="cuda"), keys["qidx"])
    q = G.normal_bf16_(torch.empty(b, h, 512, dtype=torch.bfloat16, device="cuda"), keys["q"])
    idx, cnt = K.index_topk(qidx, K.Cache(0, kidx, None, 128), n, k)
    out = K.sparse_decode(q, K.Cache(0, comp), K.Cache(0, window), idx, n, win, t, 512 ** -0.5, out_fp32=True)

    # oracle from the raw states
    r = OF.bf16_bits_to_f64(D.normal_bf16(keys["raw"], t * 512).reshape(t, 512))
    comp_ref = OF.round_bf16(OC.compress(r, w.astype(np.float64), 4, win))          # stored as bf16
    win_ref = OF.round_bf16(OR.rope(r[t - win:], np.arange(t - win, t)))
    kr = OF.bf16_bits_to_f64(D.int_bf16(keys["kidx"], n * 128).reshape(n, 128))
    qr = OF.bf16_bits_to_f64(D.int_bf16(keys["qidx"], 128))
    idx_ref, cnt_ref = OI.index_topk(qr, kr, k)
    assert int(cnt[0]) == cnt_ref == 480
    assert np.array_equal(idx[0].cpu().numpy(), idx_ref)
    qh = OF.bf16_bits_to_f64(D.normal_bf16(keys["q"], h * 512).reshape(h, 512))
    ref = OA.sparse_decode(qh[None], comp_ref[None], win_ref[None], idx_ref[None], t, 512 ** -0.5)[0]
    assert_close(to_f64(out)[0], ref)
