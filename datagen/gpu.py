"""Device-side twin of the seeded generator (libdsv4kv_datagen.so).

Fills torch CUDA tensors with exactly the bytes ``datagen`` produces on the
host for the same stream key and flat offsets, so large workloads are
generated in HBM in milliseconds and the oracle can regenerate any slice of
them on the host.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsv4kv_datagen.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m compressed_sparse_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        L.dg_normal_bf16.argtypes = [c.c_void_p, c.c_uint64, c.c_uint64, c.c_int64, c.c_void_p]
        L.dg_int_bf16.argtypes = [c.c_void_p, c.c_uint64, c.c_uint64, c.c_int64, c.c_int64, c.c_int64, c.c_void_p]
        L.dg_fp4_index_keys.argtypes = [c.c_void_p, c.c_void_p, c.c_uint64, c.c_uint64, c.c_int64, c.c_int,
                                        c.c_void_p]
        for f in (L.dg_normal_bf16, L.dg_int_bf16, L.dg_fp4_index_keys):
            f.restype = c.c_int
        _lib = L
    return _lib


def _s():
    return torch.cuda.current_stream().cuda_stream


def _ok(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{what}: CUDA error {rc}")


def normal_bf16_(t: torch.Tensor, key: int, offset: int = 0) -> torch.Tensor:
    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    _ok(lib().dg_normal_bf16(t.data_ptr(), key, offset, t.numel(), _s()), "dg_normal_bf16")
    return t


def int_bf16_(t: torch.Tensor, key: int, lo: int = -8, hi: int = 8, offset: int = 0) -> torch.Tensor:
    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    _ok(lib().dg_int_bf16(t.data_ptr(), key, offset, t.numel(), lo, hi, _s()), "dg_int_bf16")
    return t


def fp4_index_keys_(codes: torch.Tensor, scales: torch.Tensor, key: int, row0: int = 0) -> None:
    """codes u8 [rows][di/2], scales u8 [rows][di/16] (leading dims flattened)."""
    di = codes.shape[-1] * 2
    rows = codes.numel() // (di // 2)
    _ok(lib().dg_fp4_index_keys(codes.data_ptr(), scales.data_ptr(), key, row0, rows, di, _s()), "dg_fp4_index_keys")
