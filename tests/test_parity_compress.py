"""dsv4kv_compress against the oracle (c4a and c128a, bf16 and fp32 outputs)."""
import zlib

import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import compress as OC
from oracle import formats as OF
from tests._util import assert_bf16_rounding_of, assert_close, scaled_max_abs, to_f64

pytestmark = pytest.mark.gpu


def _raw(seed, b, t, d=512):
    import datagen.gpu as G
    key = D.stream_key(seed, D.TID_RAW_S, 0)
    return G.normal_bf16_(torch.empty(b, t, d, dtype=torch.bfloat16, device="cuda"), key), key


@pytest.mark.parametrize("kind,b,t,window,pos0", [
    ("c4a", 1, 2048, 128, 0),          # tiny c4a: 480 entries
    ("c4a", 2, 1000 + 3, 128, 0),      # ragged t
    ("c4a", 1, 4096, 0, 1 << 20),      # no window, large positions
    ("c4a", 2, 131072, 128, 12345),    # c4a t=131072: 32736 entries, 1023 blocks of 32 per sequence
    ("c128a", 2, 128 * 20 + 128 + 50, 128, 0),
    ("c128a", 1, 131072, 128, 0),      # c128a t=131072: 1023 entries
])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_compress(kind, b, t, window, pos0, out_fp32):
    s, k = (4, 8) if kind == "c4a" else (128, 128)
    raw, key = _raw(zlib.crc32(f"{kind}-{t}".encode()) % 1000, b, t)  # (a fixed seed per case)
    w = D.compress_weights(5, 0, k, 512)
    out = K.compress(raw, torch.from_numpy(w).cuda(), s, window, pos0=pos0, out_fp32=out_fp32)
    n = OC.n_entries(t, window, s)
    assert out.shape == (b, n, 512)
    got = to_f64(out)
    for bb in range(b):
        r = OF.bf16_bits_to_f64(D.normal_bf16(key, t * 512, offset=bb * t * 512).reshape(t, 512))
        ref = OC.compress(r, w.astype(np.float64), s, window, pos0=pos0)
        if out_fp32:
            assert_close(got[bb], ref, what=f"{kind} seq {bb}")
            assert np.abs(got[bb] - ref).max() < 1e-4       # fp32 accumulation of <= 128 taps
        else:
            # every stored value is a bf16 rounding of the fp32 entry; the
            # entries reach |x| ~ 5, where half a bf16 ulp exceeds 1e-2
            assert_bf16_rounding_of(got[bb], ref, what=f"{kind} seq {bb}")
            assert_close(got[bb], ref, max_abs=scaled_max_abs(ref), what=f"{kind} seq {bb}")


def test_window_rows_are_one_tap_compression():
    """K = 1, stride 1, weight 1: the entries are the raw rows rotated at their positions."""
    t, W = 3000, 128
    raw, key = _raw(3, 1, t)
    w = torch.ones(1, 512, dtype=torch.float32, device="cuda")
    win = K.compress(raw[:, t - W:].contiguous(), w, 1, 0, pos0=t - W, out_fp32=True)
    r = OF.bf16_bits_to_f64(D.normal_bf16(key, t * 512).reshape(t, 512))
    from oracle import rope as OR
    ref = OR.rope(r[t - W:], np.arange(t - W, t))
    assert_close(to_f64(win)[0], ref, max_abs=1e-5, rel_l2=1e-6)


@pytest.mark.parametrize("d,k,s,rope_dim", [
    (256, 8, 4, 64),       # c4a shape at dim 256 (one warp per entry)
    (1024, 8, 4, 128),     # dim 1024, a wider rotary part
    (512, 6, 4, 64),       # taps that are not 2 x stride
    (512, 40, 40, 64),     # stride = taps, not a multiple of 16 (one warp per entry)
    (512, 96, 96, 64),     # stride = taps = 96: the staged-weight kernel with 6 chunks
    (512, 128, 128, 0),    # c128a shape without rotary channels
])
def test_compress_other_shapes(d, k, s, rope_dim):
    """Shapes beside the two bench shapes: the one-warp-per-entry kernel and the staged-weight kernel at
    other tap counts."""
    b, t, window, pos0 = 2, 3 * 128 + 200, 128, 777
    raw, key = _raw(11 + d + k, b, t, d)
    w = D.compress_weights(9, 0, k, d)
    out = K.compress(raw, torch.from_numpy(w).cuda(), s, window, pos0=pos0, rope_dim=rope_dim, out_fp32=True)
    got = to_f64(out)
    for bb in range(b):
        r = OF.bf16_bits_to_f64(D.normal_bf16(key, t * d, offset=bb * t * d).reshape(t, d))
        ref = OC.compress(r, w.astype(np.float64), s, window, pos0=pos0, rope_dim=rope_dim)
        assert got[bb].shape == ref.shape
        assert np.abs(got[bb] - ref).max() < 1e-4
