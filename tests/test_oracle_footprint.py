"""Pins for oracle.footprint against the numbers the first page prints."""
from oracle import footprint as FP
from oracle.compress import n_entries

T1M = 2 ** 20


def _g(golden):
    return {name: (float(v), float(tol)) for name, v, tol in golden("footprints.txt")}


def _close(x, ref, tol):
    return abs(x - ref) <= tol * abs(ref) + 1e-12


def test_bf16_stack_and_v32_stack(golden):
    g = _g(golden)
    v4 = FP.stack_bytes(T1M)
    assert v4 == 10_333_111_296
    assert _close(v4 / FP.GIB, *g["v4_bf16_gib_per_1m_sequence"])
    v32 = FP.v32_stack_bytes(T1M)
    assert (576 + 128) * 2 == g["v32_bytes_per_token_per_layer"][0]
    assert _close(v32 / FP.GIB, *g["v32_gib_per_1m_sequence"])
    assert _close(v32 / v4, *g["v4_reduction_factor"])


def test_per_layer_and_entry_counts(golden):
    g = _g(golden)
    assert _close(FP.layer_bytes("c4a", T1M) / FP.MIB, *g["c4a_layer_mib_at_1m"])
    assert _close(FP.layer_bytes("c128a", T1M) / FP.MIB, *g["c128a_layer_mib_at_1m"])
    assert _close(n_entries(T1M, 128, 128), *g["c128a_entries_at_1m"])
    assert n_entries(T1M, 128, 128) <= g["c128a_entries_at_1m"][0] * 1.03
    assert g["layers_c4a"][0] + g["layers_c128a"][0] == g["layers_total"][0]


def test_quantised_caches_roughly_halve(golden):
    g = _g(golden)
    q = FP.stack_bytes(T1M, main_fmt="fp8", index_fmt="fp4")
    # 30 x (262112 x (516 + 72) + 128 x 516) + 31 x (8191 x 516 + 128 x 516)
    assert q == 30 * (262112 * 588 + 128 * 516) + 31 * (8191 * 516 + 128 * 516) == 4_758_707_844
    assert _close(FP.stack_bytes(T1M) / q, *g["fp8_fp4_extra_reduction"])


def test_one_million_is_two_to_the_twenty():
    # with 10^6 tokens the stack is 9.18 GiB, outside the page's 9.62: "1M" = 2^20
    assert not _close(FP.stack_bytes(10 ** 6) / FP.GIB, 9.62, 0.0006)
