"""Planted mistakes: each test builds a plausibly wrong variant of an oracle
function (on the CPU) and shows that the independent reference used by the
pins rejects it, so the pins are sharp enough to catch that class of error."""
import cmath

import numpy as np
import torch

from oracle import attention as A
from oracle import compress as C
from oracle import formats as F
from oracle import indexer as I
from oracle import rope as R


def _rope_matches_complex(fn):
    x = np.random.default_rng(0).normal(size=512)
    for pos in (1, 777):
        y = fn(x, pos)
        for m in (0, 5, 31):
            z = complex(x[448 + 2 * m], x[449 + 2 * m]) * cmath.exp(1j * pos * 10000.0 ** (-2 * m / 64))
            if abs(y[448 + 2 * m] - z.real) > 1e-9 or abs(y[449 + 2 * m] - z.imag) > 1e-9:
                return False
    return True


def test_rope_pin_catches_sign_and_pairing_errors():
    assert _rope_matches_complex(R.rope)
    assert not _rope_matches_complex(lambda x, p: R.rope(x, -p))                       # wrong sign
    assert not _rope_matches_complex(lambda x, p: R.rope(x, p, base=1000.0))            # wrong base

    def half_split(x, p):                                                              # other pairing
        x = np.array(x, dtype=np.float64)
        a = p * R.thetas()
        lo, hi = x[448:480].copy(), x[480:512].copy()
        x[448:480], x[480:512] = lo * np.cos(a) - hi * np.sin(a), lo * np.sin(a) + hi * np.cos(a)
        return x
    assert not _rope_matches_complex(half_split)


def _taps(fn, scheme, entry):
    s, k = (4, 8) if scheme == "c4a" else (128, 128)
    t = 128 + s * (entry + 2)
    hit = []
    for p in range(t):
        raw = np.zeros((t, 72))
        raw[p, 0] = 1.0
        if fn(raw, np.ones((k, 72)), s, 128)[entry, 0] != 0.0:
            hit.append(p)
    return hit


def test_diagram_pin_catches_shifted_taps(golden):
    def shifted(s_raw, w, stride, window):   # taps [s*i, s*i+K): one block late
        n = C.n_entries(len(s_raw), window, stride)
        out = np.zeros((n, s_raw.shape[1]))
        for i in range(n):
            for j in range(w.shape[0]):
                p = stride * i + j
                if p < len(s_raw):
                    out[i] += w[j] * s_raw[p]
        return out
    rows = golden("diagram_taps.txt")
    ok = [(_taps(lambda *a: C.compress(*a, rope_dim=64), sc, int(e)) == list(range(int(f), int(l) + 1)))
          for sc, e, f, l in rows]
    bad = [(_taps(shifted, sc, int(e)) == list(range(int(f), int(l) + 1))) for sc, e, f, l in rows]
    assert all(ok) and not all(bad)


def test_tie_pin_catches_higher_index_rule():
    def wrong(score, k):
        n = len(score)
        order = np.lexsort((-np.arange(n), -score))        # ties to the HIGHER index
        sel = np.sort(order[:min(k, n)])
        return np.concatenate([sel, -np.ones(k - len(sel), int)]), min(k, n)
    s = np.zeros(20)
    s[[3, 9, 15]] = 5.0
    assert list(I.topk(s, 5)[0]) == [0, 1, 3, 9, 15]
    assert list(wrong(s, 5)[0]) != [0, 1, 3, 9, 15]


def _sdpa_ok(fn):
    rng = np.random.default_rng(1)
    q, rows = rng.normal(size=(4, 512)), rng.normal(size=(50, 512))
    qt, kt = torch.from_numpy(q)[None], torch.from_numpy(rows)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt.clone(), scale=0.05)[0].numpy()
    return np.allclose(R.rope(fn(q, rows, 0.05, 900), 900), ref, atol=1e-12)


def test_attention_pin_catches_transposes_scale_and_rotation():
    assert _sdpa_ok(A.shared_kv_decode)

    def no_scale(q, rows, scale, t):
        return A.shared_kv_decode(q, rows, 1.0, t)

    def softmax_wrong_axis(q, rows, scale, t):
        s = scale * (q @ rows.T)
        p = np.exp(s - s.max(axis=0, keepdims=True))
        p /= p.sum(axis=0, keepdims=True)
        return R.rope(p @ rows, -t)

    def forward_rotation(q, rows, scale, t):
        return R.rope(A.attend(q, rows, rows, scale), +t)

    for bad in (no_scale, softmax_wrong_axis, forward_rotation):
        assert not _sdpa_ok(bad)


def test_format_pin_catches_round_half_away():
    pos = F.E4M3_TABLE[:0x7F]
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    lib = torch.from_numpy(mids).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(mids), lib)

    def half_away(v):                       # ties away from zero instead of to even
        a = np.abs(np.asarray(v, np.float64))
        hi = np.clip(np.searchsorted(pos, a, side="left"), 0, 126)
        lo = np.clip(hi - 1, 0, 126)
        return np.where(pos[hi] - a <= a - pos[lo], hi, lo).astype(np.uint8)
    assert not np.array_equal(half_away(mids), lib)


# ------------------------------------------------ the NEXT rows' oracle functions
def _pool_matches_brute(fn):
    rng = np.random.default_rng(21)
    # score of entry i = the number of leading ones of key i, in 60..69: ~15 pool entries per value
    keys = np.zeros((400, 128))
    for i, c in enumerate(rng.integers(60, 70, 400)):
        keys[i, :c] = 1.0
    keys[399] = 1.0                                                 # the best key, outside the pool
    q = np.ones(128)
    pool = np.sort(rng.choice(399, 150, replace=False))
    s = {int(i): float(keys[i] @ q) for i in pool}
    ranked = sorted(pool.tolist(), key=lambda i: (-s[i], i))
    assert s[ranked[39]] == s[ranked[40]]                           # the cut falls inside a group of ties
    want = sorted(ranked[:40])
    got, _ = fn(q, keys, np.concatenate([pool, [-1, -1]]), 40)
    return got[:40].tolist() == want


def test_pool_pin_catches_tie_and_padding_errors():
    assert _pool_matches_brute(I.index_topk_pool)

    def ties_to_higher(q, keys, pool, k):                          # ties broken toward the higher entry
        pool = np.asarray(pool)
        ent = pool[pool >= 0]
        sc = keys[ent] @ q
        order = np.lexsort((-ent, -sc))
        out = np.full(k, -1, dtype=np.int32)
        out[:min(k, len(ent))] = np.sort(ent[order[:k]])
        return out, min(k, len(ent))
    assert not _pool_matches_brute(ties_to_higher)

    def padding_as_entry(q, keys, pool, k):                        # -1 read as the last entry
        return I.index_topk_pool(q, keys, np.where(np.asarray(pool) < 0, len(keys) - 1, pool), k)
    assert not _pool_matches_brute(padding_as_entry)


def _fp8_rope_matches_worked_row(fn):
    x = np.zeros((1, 512), dtype=np.float32)
    x[0, 0], x[0, 1], x[0, 448], x[0, 511] = 224.0, 1.0, 1.5, -2.0
    codes, scales = fn(x)
    return (scales[0] == np.float32(0.5) and codes[0, 0] == 0x7E and codes[0, 1] == 0x40
            and list(codes[0, 448:450]) == [0xC0, 0x3F] and list(codes[0, 574:576]) == [0x00, 0xC0])


def test_fp8_rope_pin_catches_scale_and_byte_order_errors():
    assert _fp8_rope_matches_worked_row(F.quantize_fp8_rope_rows)

    def scale_over_all_channels(x):                                # amax taken over the rotary channels too
        x = np.asarray(x, dtype=np.float32).copy()
        x[:, 448:] *= 1000.0
        c, s = F.quantize_fp8_rope_rows(x)
        return c, s
    x_big = np.zeros((1, 512), dtype=np.float32)
    x_big[0, 0], x_big[0, 448] = 1.0, 5000.0
    _, good = F.quantize_fp8_rope_rows(x_big)
    amax_all = np.float32(5000.0) / np.float32(448.0)
    assert good[0] != amax_all                                      # the body's amax sets the scale

    def big_endian_rope(x):
        c, s = F.quantize_fp8_rope_rows(x)
        c = c.copy()
        c[:, 448:] = c[:, 448:].reshape(c.shape[0], -1, 2)[:, :, ::-1].reshape(c.shape[0], -1)
        return c, s
    assert not _fp8_rope_matches_worked_row(big_endian_rope)


def test_append_pin_catches_late_emission():
    """An emission rule one stride late leaves an entry missing at the step its block leaves the window."""
    def late(t, window, stride):
        return max(0, (t - window) // stride - 1)
    ok = all(C.n_entries(t + 1, 128, 4) - C.n_entries(t, 128, 4) == (1 if (t + 1 - 128) >= 4 and (t + 1 - 128) % 4 == 0 else 0)
             for t in range(400))
    bad = all(late(t + 1, 128, 4) - late(t, 128, 4) == (1 if (t + 1 - 128) >= 4 and (t + 1 - 128) % 4 == 0 else 0)
              for t in range(400))
    assert ok and not bad
