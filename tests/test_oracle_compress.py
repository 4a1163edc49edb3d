"""Pins for oracle.rope and oracle.compress.

Independent references: the tap sets printed in the walkthrough's Step 4
diagrams (tests/golden/diagram_taps.txt), complex-number rotation from the
Python standard library, strided subsampling, numpy block means, linearity.
"""
import cmath

import numpy as np
import pytest

from oracle import compress as C
from oracle import rope as R


def test_thetas_closed_form():
    th = R.thetas(64, 10000.0)
    assert th[0] == 1.0
    assert np.isclose(th[1], 10000.0 ** (-2 / 64), rtol=0, atol=1e-15)
    assert np.isclose(th[31], 10000.0 ** (-62 / 64), rtol=1e-14)


def test_rope_against_complex_rotation():
    rng = np.random.default_rng(0)
    x = rng.normal(size=512)
    for pos in (0, 1, 7, 2048, 131071, 1048576, -1048576):
        y = R.rope(x, pos)
        assert np.array_equal(y[:448], x[:448])           # non-rotary channels untouched
        for m in (0, 1, 13, 31):
            z = complex(x[448 + 2 * m], x[449 + 2 * m]) * cmath.exp(1j * pos * 10000.0 ** (-2 * m / 64))
            assert abs(y[448 + 2 * m] - z.real) < 1e-9 and abs(y[449 + 2 * m] - z.imag) < 1e-9


def test_rope_invariants():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(4, 512))
    assert np.array_equal(R.rope(x, 0), x)
    y = R.rope(x, 12345)
    assert np.allclose(R.rope(y, -12345), x, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # relative position: <rope(q,t), rope(k,p)> depends only on t - p
    q, k = x[0], x[1]
    d1 = R.rope(q, 1000) @ R.rope(k, 900)
    d2 = R.rope(q, 5100) @ R.rope(k, 5000)
    assert abs(d1 - d2) < 1e-9
    # composition
    assert np.allclose(R.rope(R.rope(x, 37), 5), R.rope(x, 42), atol=1e-12)


@pytest.mark.parametrize("t,w,s,n", [
    (2048, 128, 4, 480), (131072, 128, 128, 1023), (131072, 128, 4, 32736),
    (1048576, 128, 4, 262112), (1048576, 128, 128, 8191),
    (262144, 128, 4, 65504), (262144, 128, 128, 2047),
    (128, 128, 4, 0), (100, 128, 4, 0), (131, 128, 4, 0), (132, 128, 4, 1),
])
def test_entry_counts(t, w, s, n):
    assert C.n_entries(t, w, s) == n


def test_diagram_tap_sets(golden):
    """Impulse responses of the compressor reproduce the walkthrough's tap sets."""
    for scheme, entry, first, last in golden("diagram_taps.txt"):
        entry, first, last = int(entry), int(first), int(last)
        s, k = (4, 8) if scheme == "c4a" else (128, 128)
        t = 128 + s * (entry + 2)
        w = np.full((k, 8 + 64), 1.0)                # D = 72: 8 plain + 64 rotary channels
        hit = []
        for p in range(t):
            raw = np.zeros((t, 72))
            raw[p, 0] = 1.0
            out = C.compress(raw, w, s, 128)
            if out[entry, 0] != 0.0:
                hit.append(p)
        assert hit == list(range(first, last + 1)), (scheme, entry)


def test_one_hot_weights_are_strided_subsampling():
    rng = np.random.default_rng(2)
    for s, k in ((4, 8), (128, 128)):
        t = 128 + s * 9
        raw = rng.normal(size=(t, 512))
        w = np.zeros((k, 512))
        w[k - s] = 1.0
        out = C.compress(raw, w, s, 128)
        n = C.n_entries(t, 128, s)
        assert out.shape == (n, 512)
        for i in range(n):
            assert np.array_equal(out[i], R.rope(raw[s * i], s * i))


def test_uniform_weights_are_block_means():
    rng = np.random.default_rng(3)
    raw = rng.normal(size=(128 + 128 * 3, 512))
    out = C.compress(raw, np.full((128, 512), 1 / 128), 128, 128, rope_dim=64)
    for i in range(3):
        assert np.allclose(out[i], R.rope(raw[128 * i:128 * i + 128].mean(axis=0), 128 * i), atol=1e-13)
    # c4a: entry 0 sees 4 live taps and 4 zero taps (no renormalisation)
    raw = rng.normal(size=(128 + 40, 512))
    out = C.compress(raw, np.full((8, 512), 1 / 8), 4, 128)
    assert np.allclose(out[0], R.rope(raw[0:4].sum(axis=0) / 8, 0), atol=1e-13)
    assert np.allclose(out[3], R.rope(raw[8:16].mean(axis=0), 12), atol=1e-13)


def test_linearity_in_weights_and_pos0():
    rng = np.random.default_rng(4)
    raw = rng.normal(size=(128 + 64, 512))
    w1, w2 = rng.normal(size=(8, 512)), rng.normal(size=(8, 512))
    lhs = C.compress(raw, 2.0 * w1 - 0.5 * w2, 4, 128)
    rhs = 2.0 * C.compress(raw, w1, 4, 128) - 0.5 * C.compress(raw, w2, 4, 128)
    assert np.allclose(lhs, rhs, atol=1e-12)
    shifted = C.compress(raw, w1, 4, 128, pos0=1000)
    assert np.allclose(shifted, R.rope(C.compress(raw, w1, 4, 128), 1000), atol=1e-12)


def test_per_channel_weights_are_not_transposed():
    rng = np.random.default_rng(5)
    raw = rng.normal(size=(128 + 8, 16 + 64))
    w = rng.normal(size=(8, 80))
    out = C.compress(raw, w, 4, 128, rope_dim=64)
    # channel 3 of entry 1 = sum_j w[j,3] * raw[j,3] (taps 0..7), plain channel so no rotation
    assert np.isclose(out[1, 3], sum(w[j, 3] * raw[j, 3] for j in range(8)), atol=1e-13)


# ------------------------------------------------ incremental maintenance
@pytest.mark.parametrize("stride,k_taps,window", [(4, 8, 128), (128, 128, 128), (4, 8, 0), (8, 16, 20)])
def test_append_emits_each_entry_when_its_block_leaves_the_window(stride, k_taps, window):
    """Entry count grows by one exactly when (t+1-W) reaches a multiple of the
    stride, and the new entry's taps all lie in the last W + K positions (the
    raw ring the incremental kernel keeps)."""
    prev = 0
    for t in range(0, 6 * stride + window + 3):
        n1 = C.n_entries(t + 1, window, stride)
        grew = n1 - prev
        assert grew in (0, 1)
        assert grew == (1 if (t + 1 - window) >= stride and (t + 1 - window) % stride == 0 else 0)
        if grew:
            taps = C.tap_positions(n1 - 1, stride, k_taps)
            live = taps[taps >= 0]
            assert live.min() >= t + 1 - window - k_taps and live.max() <= t - window
        prev = n1


def test_append_state_is_the_whole_history_compressed():
    rng = np.random.default_rng(12)
    s = rng.standard_normal((300, 64))
    w = rng.random((8, 64))
    pos, win, ent = C.append_state(s, w, 4, 32, rope_dim=16)
    assert pos.tolist() == list(range(268, 300))
    assert np.allclose(win[5], R.rope(s[273], 273, 16), rtol=0, atol=1e-12)
    assert ent.shape == (67, 64)                      # floor((300 - 32) / 4)
    # entry 10 mixes positions 36..43 (taps 4*10 + 4 - 8 + j), rotated at 40
    raw = sum(w[j] * s[36 + j] for j in range(8))
    assert np.allclose(ent[10], R.rope(raw, 40, 16), rtol=0, atol=1e-12)
