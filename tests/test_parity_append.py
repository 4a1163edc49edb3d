"""dsv4kv_append (incremental cache maintenance, one call per decoded token)
against the oracle's whole-history caches and the batch compressor."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import compress as OC
from oracle import formats as OF
from oracle import rope as OR
from tests._util import assert_close, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stride,k_taps,window,steps,b", [
    (4, 8, 128, 700, 2),          # c4a: 143 entries emitted one step at a time
    (128, 128, 128, 1300, 2),     # c128a: 9 entries, 128 taps each
    (4, 8, 0, 90, 1),             # no window: the newest state is a tap
    (4, 8, 128, 100, 1),          # fewer steps than the window: no entry yet
])
def test_append_reaches_the_whole_history_caches(stride, k_taps, window, steps, b):
    import datagen.gpu as G
    key = D.stream_key(300 + stride + window, D.TID_RAW_S, 0)
    s = G.normal_bf16_(torch.empty(b, steps, 512, dtype=torch.bfloat16, device="cuda"), key)
    w_np = D.compress_weights(9, 0, k_taps, 512)
    w = torch.from_numpy(w_np).cuda()
    ring = window + k_taps
    raw = torch.zeros(b, ring, 512, dtype=torch.bfloat16, device="cuda")
    win = torch.zeros(b, max(window, 1), 512, dtype=torch.bfloat16, device="cuda")
    n = OC.n_entries(steps, window, stride)
    comp = torch.zeros(b, n + 2, 512, dtype=torch.bfloat16, device="cuda")
    for t in range(steps):
        K.append(s[:, t].contiguous(), w, t, stride, window, raw, win if window else None, comp)
    torch.cuda.synchronize()
    got_c, got_w, got_r = to_f64(comp), to_f64(win), to_f64(raw)
    batch = to_f64(K.compress(s, w, stride, window)) if n else np.zeros((b, 0, 512))
    for bb in range(b):
        hist = OF.bf16_bits_to_f64(D.normal_bf16(key, steps * 512, offset=bb * steps * 512).reshape(steps, 512))
        pos, wrows, ents = OC.append_state(hist, w_np.astype(np.float64), stride, window)
        assert ents.shape[0] == n
        # the caches are bf16: compare with the oracle's values rounded to bf16
        if n:
            assert_close(got_c[bb, :n], OF.round_bf16(ents), what=f"entries seq {bb}")
            # against the batch compressor: the same fp32 sums up to their order (<= one bf16 step)
            assert np.all(np.abs(got_c[bb, :n] - batch[bb]) <= 2.0 ** -7 * np.maximum(np.abs(batch[bb]), 2.0 ** -100))
        assert np.all(got_c[bb, n:] == 0)                # nothing beyond the entries due
        for i, p in enumerate(pos):
            assert_close(got_w[bb, p % window], OF.round_bf16(wrows[i]), what=f"window row of position {p}")
        for p in range(max(0, steps - ring), steps):     # the raw ring holds the last W + K states exactly
            assert np.array_equal(got_r[bb, p % ring], hist[p])


def test_append_rejects_an_entry_beyond_the_cache():
    b = 1
    w = torch.ones(8, 512, device="cuda")
    raw = torch.zeros(b, 136, 512, dtype=torch.bfloat16, device="cuda")
    win = torch.zeros(b, 128, 512, dtype=torch.bfloat16, device="cuda")
    comp = torch.zeros(b, 1, 512, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(b, 512, dtype=torch.bfloat16, device="cuda")
    K.append(x, w, 131, 4, 128, raw, win, comp)          # entry 0 becomes due at t + 1 = 132
    with pytest.raises(K.Dsv4kvError):
        K.append(x, w, 135, 4, 128, raw, win, comp)      # entry 1 would not fit one row
