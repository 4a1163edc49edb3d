"""The shared input generator: determinism, slicing, distributions."""
import numpy as np

import datagen as D


def test_splitmix64_reference_value():
    # SplitMix64 from state 0: first output 0xE220A8397B1DCDAF (published test vector)
    assert D._py_mix64(0x9E3779B97F4A7C15) == 0xE220A8397B1DCDAF
    assert int(D._mix64(np.array([0x9E3779B97F4A7C15], dtype=np.uint64))[0]) == 0xE220A8397B1DCDAF


def test_streams_are_deterministic_and_sliceable():
    k = D.stream_key(1234, D.TID_COMP, 3)
    a = D.normal_bf16(k, 5000)
    assert np.array_equal(a, D.normal_bf16(k, 5000))
    assert np.array_equal(a[1000:2000], D.normal_bf16(k, 1000, offset=1000))
    rows = np.array([7, 2, 9])
    r = D.rows_normal_bf16(k, rows, 500)
    assert np.array_equal(r[1], a[1000:1500])
    assert not np.array_equal(a, D.normal_bf16(D.stream_key(1234, D.TID_COMP, 4), 5000))


def test_normal_moments():
    k = D.stream_key(1, D.TID_RAW_S)
    x = D.normal_values(k, np.arange(1 << 20, dtype=np.uint64))
    assert abs(x.mean()) < 0.005 and abs(x.var() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0


def test_uniform_ints():
    k = D.stream_key(2, D.TID_KIDX)
    v = D.uniform_int(k, 170000, -8, 8)
    assert v.min() == -8 and v.max() == 8
    freq = np.bincount(v + 8) / len(v)
    assert np.all(np.abs(freq - 1 / 17) < 0.003)


def test_fp4_index_keys_dequantise_to_small_integers():
    codes, scales = D.fp4_index_keys_rows(D.stream_key(3, D.TID_KIDX_FP4), np.arange(100), 128)
    assert codes.shape == (100, 64) and scales.shape == (100, 8)
    lo, hi = codes & 0xF, codes >> 4
    for nib in (lo, hi):
        assert np.all((nib & 7) <= 6)
    vals = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0}
    mag = np.array(sorted(vals))[np.concatenate([lo & 7, hi & 7]).ravel()] * 2.0
    assert set(np.unique(mag)) <= {0, 1, 2, 3, 4, 6, 8}


def test_compress_weights_are_softmax_normalised():
    w = D.compress_weights(9, 0, 8, 512)
    assert w.dtype == np.float32 and w.shape == (8, 512)
    assert np.all(w > 0) and np.allclose(w.astype(np.float64).sum(axis=0), 1.0, atol=1e-6)
