"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/dsv4kv.h declares, sizes its workspaces, and
rejects bad arguments with status codes (nothing is launched)."""
import ctypes
import os
import re

import pytest

import compressed_sparse_kv_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "dsv4kv.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dsv4kv_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = K.lib()
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) <= set(K._SIGS)      # the binding declares a signature for each


def test_version_and_entry_counts():
    assert K.lib().dsv4kv_version().startswith(b"dsv4kv")
    assert K.compress_entries(2048, 128, 4) == 480
    assert K.compress_entries(131072, 128, 128) == 1023
    assert K.compress_entries(1 << 20, 128, 4) == 262112
    assert K.compress_entries(100, 128, 4) == 0


def test_workspace_sizes_grow_with_the_problem():
    a = K.index_topk_workspace_bytes(1, 1000, 512)
    b = K.index_topk_workspace_bytes(32, 32736, 512)
    assert 0 < a < b
    assert K.sparse_decode_workspace_bytes(32, 64, 512, 128) > 0
    assert K.dense_decode_workspace_bytes(8, 64, 1023, 128) > 0
    assert K.index_topk_workspace_bytes(1, 10, 0) == 0           # invalid k


def _status(rc):
    return rc, K.lib().dsv4kv_last_error().decode()


def test_bad_arguments_return_status_codes():
    L = K.lib()
    z = ctypes.c_void_p(0)
    # compress: bad stride
    rc, msg = _status(L.dsv4kv_compress(z, z, 1, 2048, 512, 8, 0, 128, 0, 64, 1e4, 0, z, z))
    assert rc == 1 and "compress" in msg
    # compress: odd rope_dim
    assert L.dsv4kv_compress(z, z, 1, 2048, 512, 8, 4, 128, 0, 63, 1e4, 0, z, z) == 1
    # compress: null pointers with work to do
    assert L.dsv4kv_compress(z, z, 1, 2048, 512, 8, 4, 128, 0, 64, 1e4, 0, z, z) == 1
    # compress: nothing to do is OK without touching pointers
    assert L.dsv4kv_compress(z, z, 1, 100, 512, 8, 4, 128, 0, 64, 1e4, 0, z, z) == 0
    # quantize: bf16 is not a quantised format
    assert L.dsv4kv_quantize(z, 0, 10, 512, 0, z, z, z) == 2
    assert L.dsv4kv_quantize(z, 0, 10, 512, 1, z, z, z) == 1
    # index_topk
    keys = K.CacheDesc(0, 128, 1000, None, None)
    assert L.dsv4kv_index_topk(z, ctypes.byref(keys), 1, 1000, 0, z, z, z, 0, z) == 2       # k = 0
    assert L.dsv4kv_index_topk(z, ctypes.byref(keys), 1, 1000, 4096, z, z, z, 0, z) == 2    # k too big
    bad_dim = K.CacheDesc(0, 64, 1000, 16, None)
    assert L.dsv4kv_index_topk(16, ctypes.byref(bad_dim), 1, 1000, 512, 16, z, 16, 1 << 30, z) == 2
    odd = K.CacheDesc(0, 128, 1000, 8, None)                                              # misaligned
    assert L.dsv4kv_index_topk(16, ctypes.byref(odd), 1, 1000, 512, 16, z, 16, 1 << 30, z) == 1
    short = K.CacheDesc(0, 128, 10, 16, None)                                             # rows < n
    assert L.dsv4kv_index_topk(16, ctypes.byref(short), 1, 1000, 512, 16, z, 16, 1 << 30, z) == 1
    good = K.CacheDesc(0, 128, 1000, 16, None)
    assert L.dsv4kv_index_topk(16, ctypes.byref(good), 1, 1000, 512, 16, z, 16, 64, z) == 3  # workspace
    fp8 = K.CacheDesc(1, 128, 1000, 16, 16)
    assert L.dsv4kv_index_topk(16, ctypes.byref(fp8), 1, 1000, 512, 16, z, 16, 1 << 30, z) == 2
    # decode
    comp = K.CacheDesc(0, 512, 100, 16, None)
    win = K.CacheDesc(0, 512, 128, 16, None)
    assert L.dsv4kv_dense_decode(16, ctypes.byref(comp), ctypes.byref(win), 1, 65, 100, 128, 2048, 0.04, 64, 1e4,
                                 0, 16, 16, 1 << 30, z) == 2                                  # heads > 64
    assert L.dsv4kv_dense_decode(16, ctypes.byref(comp), ctypes.byref(win), 1, 16, 100, 128, 2048, 0.04, 64, 1e4,
                                 0, 16, 16, 8, z) == 3                                        # workspace
    assert L.dsv4kv_dense_decode(16, ctypes.byref(comp), ctypes.byref(win), 1, 16, 101, 128, 2048, 0.04, 64, 1e4,
                                 0, 16, 16, 1 << 30, z) == 1                                  # comp rows < n
    d256 = K.CacheDesc(0, 256, 100, 16, None)
    assert L.dsv4kv_dense_decode(16, ctypes.byref(d256), ctypes.byref(win), 1, 16, 100, 128, 2048, 0.04, 64, 1e4,
                                 0, 16, 16, 1 << 30, z) == 2                                  # dim != 512
    assert L.dsv4kv_sparse_decode(16, ctypes.byref(comp), ctypes.byref(win), z, 1, 16, 100, 128, 512, 2048, 0.04,
                                  64, 1e4, 0, 16, 16, 1 << 30, z) == 1                        # idx null
    assert L.dsv4kv_sparse_decode(16, ctypes.byref(comp), ctypes.byref(win), 16, 1, 16, 100, 128, 4096, 2048, 0.04,
                                  64, 1e4, 0, 16, 16, 1 << 30, z) == 2                        # k too big


def test_new_entry_points_reject_bad_arguments():
    """dsv4kv_index_topk_pool, dsv4kv_append and the fp8 + bf16-rotary format
    answer bad arguments with status codes before any launch."""
    L = K.lib()
    z = ctypes.c_void_p(0)
    keys = K.CacheDesc(0, 128, 1000, 16, None)
    pool_args = lambda k, cap, ws: (16, ctypes.byref(keys), 1, 1000, 16, cap, k, 16, z, 16, ws, z)
    assert L.dsv4kv_index_topk_pool(*pool_args(0, 64, 16)) == 2              # k = 0
    assert L.dsv4kv_index_topk_pool(*pool_args(512, 9000, 16)) == 2          # pool beyond 8192
    assert L.dsv4kv_index_topk_pool(*pool_args(512, 64, 8)) == 3             # workspace too small
    fp8 = K.CacheDesc(1, 128, 1000, 16, 16)
    assert L.dsv4kv_index_topk_pool(16, ctypes.byref(fp8), 1, 1000, 16, 64, 512, 16, z, 16, 16, z) == 2
    assert L.dsv4kv_index_topk_pool(16, ctypes.byref(keys), 0, 1000, 16, 64, 512, 16, z, 16, 16, z) == 0  # no batch
    assert K.lib().dsv4kv_index_topk_pool_workspace_bytes(4, 2048, 512) == 16
    # append: bad stride, odd rope_dim, a window ring missing, an entry beyond the cache
    assert L.dsv4kv_append(16, 16, 1, 0, 512, 8, 0, 128, 64, 1e4, 16, 16, 16, 10, z) == 1
    assert L.dsv4kv_append(16, 16, 1, 0, 512, 8, 4, 128, 63, 1e4, 16, 16, 16, 10, z) == 1
    assert L.dsv4kv_append(16, 16, 1, 0, 512, 8, 4, 128, 64, 1e4, 16, z, 16, 10, z) == 1
    rc, msg = _status(L.dsv4kv_append(16, 16, 1, 135, 512, 8, 4, 128, 64, 1e4, 16, 16, 16, 1, z))
    assert rc == 1 and "does not fit" in msg
    assert L.dsv4kv_append(z, z, 0, 5, 512, 8, 4, 128, 64, 1e4, z, z, z, 0, z) == 0   # empty batch
    # the fp8 + bf16-rotary format needs rope_dim == 64 in the decode calls
    f3 = K.CacheDesc(3, 512, 100, 16, 16)
    rc = L.dsv4kv_dense_decode(16, ctypes.byref(f3), ctypes.byref(f3), 1, 64, 100, 100, 4096, 0.044, 32, 1e4, 0,
                               16, 16, 1 << 30, z)
    assert rc == 2 and "rope_dim" in K.lib().dsv4kv_last_error().decode()


def test_selftest_rejects_a_null_status():
    """The bounded-wait self-test validates its argument on the host (nothing launched)."""
    z = ctypes.c_void_p(0)
    rc, msg = _status(K.lib().dsv4kv_selftest_wait_timeout(z, z))
    assert rc == 1 and "status" in msg
