"""Pins for oracle.formats: OCP code tables, rounding, quantisers.

Independent references: values fixed by the OCP 8-bit floating point and
Microscaling specs, torch's own float8_e4m3fn conversion (a library routine),
brute-force nearest-value search, and closed-form error bounds.
"""
import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e4m3_table_known_values():
    t = F.E4M3_TABLE
    assert t[0x00] == 0.0 and np.signbit(t[0x80])
    assert t[0x01] == 2.0 ** -9            # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert t[0x08] == 2.0 ** -6            # smallest normal
    assert t[0x38] == 1.0
    assert t[0x40] == 2.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)        # codes 0..126 increase


def test_e4m3_table_matches_torch_decode():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(lib) & np.isnan(F.E4M3_TABLE)
    assert np.all(both_nan | (lib == F.E4M3_TABLE))


def test_e2m1_table():
    assert list(F.E2M1_TABLE[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(F.E2M1_TABLE[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def _brute_nearest_even(v, table_pos):
    """Reference by exhaustive search over codes."""
    out = []
    for x in v:
        a = abs(x)
        if a >= table_pos[-1]:
            c = len(table_pos) - 1
        else:
            d = np.abs(table_pos - a)
            best = np.flatnonzero(d == d.min())
            c = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        out.append(c)
    return np.array(out)


def test_e4m3_encode_matches_torch_cast_and_brute_force():
    rng = np.random.default_rng(1)
    pos = F.E4M3_TABLE[:0x7F]
    mids = (pos[1:] + pos[:-1]) / 2
    x = np.concatenate([
        rng.uniform(-463, 463, 4000), rng.normal(0, 1, 4000), rng.normal(0, 0.01, 2000),
        mids, -mids, pos, -pos, [0.0, -0.0, 1e-30, -1e-30],
    ]).astype(np.float32)
    ours = F.e4m3_encode(x)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)
    brute = _brute_nearest_even(x.astype(np.float64), pos)
    assert np.array_equal(ours & 0x7F, brute)


def test_e4m3_saturates():
    x = np.array([448.0, 464.0, 500.0, 1e30, -1e30], dtype=np.float32)
    assert list(F.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_e2m1_encode_brute_force_and_ties():
    pos = F.E2M1_TABLE[:8]
    mids = (pos[1:] + pos[:-1]) / 2      # .25 .75 1.25 1.75 2.5 3.5 5
    x = np.concatenate([np.linspace(-7, 7, 561), mids, -mids, pos]).astype(np.float32)
    ours = F.e2m1_encode(x)
    assert np.array_equal(ours & 0x7, _brute_nearest_even(x.astype(np.float64), pos))
    # ties go to the even code: 0.25->0, 0.75->1.0(code2), 1.25->1.0, 1.75->2.0, 2.5->2.0, 3.5->4.0, 5->4.0
    assert list(F.e2m1_encode(mids.astype(np.float32))) == [0, 2, 2, 4, 4, 6, 6]
    assert F.e2m1_encode(np.float32([7.0]))[0] == 7          # saturates at 6


def test_bf16_rounding_matches_torch_on_f32_values():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.normal(0, 3, 10000), rng.normal(0, 1e-30, 100)]).astype(np.float32)
    ours = F.f64_to_bf16_bits(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)
    assert np.array_equal(F.bf16_bits_to_f64(lib), torch.from_numpy(lib.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_fp8_row_quantiser():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (64, 512)).astype(np.float32)
    codes, scale = F.quantize_fp8_rows(x)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scale, (amax / np.float32(448)).astype(np.float32))
    # the element of largest magnitude lands on +-448
    j = np.abs(x).argmax(axis=1)
    assert np.all((codes[np.arange(64), j] & 0x7F) == 0x7E)
    deq = F.dequant_fp8_rows(codes, scale)
    q = x / scale[:, None]
    # error bound: half an E4M3 spacing at |q| (spacing 2^(e-3), 2^-9 in the subnormal range)
    e = np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6)))
    half_ulp = 0.5 * 2.0 ** (e - 3) * scale[:, None]
    assert np.all(np.abs(deq - x) <= half_ulp * (1 + 1e-6))
    z_codes, z_scale = F.quantize_fp8_rows(np.zeros((2, 512), np.float32))
    assert np.all(z_codes == 0) and np.all(z_scale == 1.0)


def test_fp4_group_quantiser():
    rng = np.random.default_rng(4)
    x = rng.normal(0, 1, (32, 512)).astype(np.float32)
    codes, sc = F.quantize_fp4_rows(x)
    assert codes.shape == (32, 256) and sc.shape == (32, 32)
    s = F.E4M3_TABLE[sc]
    amax = np.abs(x.reshape(32, 32, 16)).max(-1)
    assert np.array_equal(sc, F.e4m3_encode((amax / np.float32(6)).astype(np.float32)))
    deq = F.dequant_fp4_rows(codes, sc)
    q = (x.reshape(32, 32, 16) / s[..., None].astype(np.float32)).reshape(32, 512)
    # half an E2M1 spacing at |q| (0.25 below 2, 0.5 below 4, 1 above), or the saturation gap
    aq = np.abs(q)
    half = np.where(aq < 2, 0.25, np.where(aq < 4, 0.5, 1.0))
    sat = np.maximum(aq - 6.0, 0.0)
    bound = (half + sat) * np.repeat(s, 16, axis=1)
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-6))


def test_fp4_representable_values_round_trip():
    rng = np.random.default_rng(5)
    nib = rng.integers(0, 16, (8, 512)).astype(np.uint8)
    nib[:, ::16] = 7                                  # every group reaches amax 6 * 2
    x = (F.E2M1_TABLE[nib] * 2.0).astype(np.float32)  # scale 2.0 is exact in E4M3
    codes, sc = F.quantize_fp4_rows(x)
    assert np.all(F.E4M3_TABLE[sc] == 2.0)
    assert np.array_equal(F.dequant_fp4_rows(codes, sc), x.astype(np.float64))
    # packing: even channel in the low nibble
    assert np.array_equal(F.unpack_fp4(codes) & 7, nib & 7)


def test_fp4_zero_group_and_underflowing_scale():
    x = np.zeros((1, 32), np.float32)
    x[0, 16:] = 1e-6                     # amax/6 underflows E4M3 (min 2^-9)
    codes, sc = F.quantize_fp4_rows(x)
    assert np.all(sc == 0) and np.all(codes == 0)


# ------------------------------------------------ fp8 body + bf16 rotary channels
def test_fp8_rope_worked_example():
    """A row worked by hand: body amax 224 -> scale 0.5; 224 / 0.5 = 448 is
    code 0x7E, 1 / 0.5 = 2 is code 0x40; rotary 1.5 is bf16 0x3FC0 and -2 is
    0xC000, stored little-endian after the 448 code bytes."""
    x = np.zeros((1, 512), dtype=np.float32)
    x[0, 0], x[0, 1], x[0, 447] = 224.0, 1.0, -0.25
    x[0, 448], x[0, 511] = 1.5, -2.0
    codes, scales = F.quantize_fp8_rope_rows(x)
    assert codes.shape == (1, 576) and codes.dtype == np.uint8
    assert scales[0] == np.float32(0.5)
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0x40
    assert codes[0, 447] == 0xB0                      # -0.5 = -(1.0 * 2^-1): S=1, E=6, M=0
    assert list(codes[0, 448:450]) == [0xC0, 0x3F]     # 1.5 -> 0x3FC0
    assert list(codes[0, 574:576]) == [0x00, 0xC0]     # -2.0 -> 0xC000
    assert np.all(codes[0, 2:447] == 0) and np.all(codes[0, 450:574] == 0)
    back = F.dequant_fp8_rope_rows(codes, scales)
    assert back[0, 0] == 224.0 and back[0, 1] == 1.0 and back[0, 447] == -0.25
    assert back[0, 448] == 1.5 and back[0, 511] == -2.0


def test_fp8_rope_rotary_channels_do_not_set_the_scale():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((8, 512)).astype(np.float32)
    x[:, 448:] *= 1000.0                                # large rotary values
    codes, scales = F.quantize_fp8_rope_rows(x)
    amax = np.max(np.abs(x[:, :448]), axis=1)
    assert np.array_equal(scales, (amax / np.float32(448.0)).astype(np.float32))
    back = F.dequant_fp8_rope_rows(codes, scales)
    ref = torch.from_numpy(x[:, 448:]).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(back[:, 448:], ref)           # rotary: bf16, nearest even (torch cast)


def test_fp8_rope_body_error_bound_and_zero_rows():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((64, 512)) * rng.uniform(0.01, 50, (64, 1))).astype(np.float32)
    x[3, :448] = 0.0
    codes, scales = F.quantize_fp8_rope_rows(x)
    assert scales[3] == 1.0 and np.all(codes[3, :448] == 0)
    back = F.dequant_fp8_rope_rows(codes, scales)
    # |q - x/s| <= half the E4M3 spacing at |x/s| (2^(e-3) / 2 for normals, 2^-10 below 2^-6)
    q = x[:, :448] / scales[:, None]
    e = np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6)))
    half = 2.0 ** (e - 4)
    assert np.all(np.abs(back[:, :448] / scales[:, None].astype(np.float64) - q) <= half * (1 + 1e-12))
