"""dsv4kv_quantize against the oracle: codes and scales bit-exact."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_b200 as K
import datagen as D
from oracle import formats as OF
from tests._util import from_bits

pytestmark = pytest.mark.gpu


def _special_rows(d):
    rng = np.random.default_rng(d)
    rows = [np.zeros(d), -np.zeros(d), np.full(d, 1e-30), rng.normal(0, 1e-3, d), rng.normal(0, 1e4, d)]
    tie = np.zeros(d)
    tie[:8] = [448.0, 1.0625, 1.1875, -1.0625, 3.0, 5.0, -5.0, 0.25]   # E4M3/E2M1 ties after scaling
    rows.append(tie)
    return np.stack(rows)


@pytest.mark.parametrize("fmt", [K.FP8_E4M3_ROW, K.FP4_E2M1_G16, K.FP8_E4M3_ROW_ROPE_BF16])
@pytest.mark.parametrize("d", [128, 512])
@pytest.mark.parametrize("in_fp32", [False, True])
def test_quantize_bit_exact(fmt, d, in_fp32):
    rows = 3000 + 7
    key = D.stream_key(21, D.TID_STATES, d)
    bits = D.normal_bf16(key, rows * d).reshape(rows, d)
    x = OF.bf16_bits_to_f64(bits)
    x = np.concatenate([x, _special_rows(d)])
    if in_fp32:
        xin = torch.from_numpy(x.astype(np.float32)).cuda()
        x32 = x.astype(np.float32)
    else:
        b16 = OF.f64_to_bf16_bits(x)
        xin = from_bits(b16)
        x32 = OF.bf16_bits_to_f64(b16).astype(np.float32)
    codes, scales = K.quantize(xin, fmt)
    if fmt == K.FP8_E4M3_ROW:
        rc, rs = OF.quantize_fp8_rows(x32)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    elif fmt == K.FP8_E4M3_ROW_ROPE_BF16:
        rc, rs = OF.quantize_fp8_rope_rows(x32)
        assert codes.shape[-1] == d + 64
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    else:
        rc, rs = OF.quantize_fp4_rows(x32)
        assert np.array_equal(scales.cpu().numpy(), rs)
    got = codes.cpu().numpy()
    bad = np.argwhere(got != rc)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}: {got[tuple(bad[0])]:#x} vs {rc[tuple(bad[0])]:#x}"


def test_quantize_full_size_rows():
    """fp8 and fp4 over 64 x 2175 rows of 512 (the quantised c128a cache shape)."""
    import datagen.gpu as G
    rows = 64 * 2175
    key = D.stream_key(8, D.TID_STATES, 0)
    x = G.normal_bf16_(torch.empty(rows, 512, dtype=torch.bfloat16, device="cuda"), key)
    for fmt in (K.FP8_E4M3_ROW, K.FP4_E2M1_G16):
        codes, scales = K.quantize(x, fmt)
        sample = np.array([0, 1, 4097, rows - 1])
        x32 = OF.bf16_bits_to_f64(D.rows_normal_bf16(key, sample, 512)).astype(np.float32)
        rc, rs = (OF.quantize_fp8_rows if fmt == K.FP8_E4M3_ROW else OF.quantize_fp4_rows)(x32)
        assert np.array_equal(codes[sample].cpu().numpy(), rc)
        got_s = scales[sample].cpu().numpy()
        assert np.array_equal(got_s.view(np.uint8), np.asarray(rs).view(np.uint8))


@pytest.mark.parametrize("fmt", [K.FP8_E4M3_ROW, K.FP4_E2M1_G16, K.FP8_E4M3_ROW_ROPE_BF16])
def test_quantize_bit_exact_across_magnitudes(fmt):
    """fp32 rows of uniform values whose magnitudes span 2^-100 .. 2^60, so that the row scales run
    from far below 2^-64 (where a reciprocal of the scale would overflow) to far above 1, and the
    quotients by the scale land everywhere between grid points: a quotient off the correctly
    rounded x / scale by one unit in the last place changes a code about once in 2^20 values."""
    rng = np.random.default_rng(5)
    rows, d = 20000, 512
    mag = np.exp2(rng.uniform(-100, 60, size=(rows, 1)))
    x32 = (rng.uniform(-1, 1, size=(rows, d)) * mag).astype(np.float32)
    codes, scales = K.quantize(torch.from_numpy(x32).cuda(), fmt)
    if fmt == K.FP8_E4M3_ROW:
        rc, rs = OF.quantize_fp8_rows(x32)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    elif fmt == K.FP8_E4M3_ROW_ROPE_BF16:
        rc, rs = OF.quantize_fp8_rope_rows(x32)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    else:
        rc, rs = OF.quantize_fp4_rows(x32)
        assert np.array_equal(scales.cpu().numpy(), rs)
    got = codes.cpu().numpy()
    assert np.array_equal(got, rc), f"{int((got != rc).sum())} codes differ"
