"""Python binding of libdsv4kv (C ABI in include/dsv4kv.h).

Argument marshalling only: every step of the path runs in the library's
sm_100a kernels.  PyTorch provides device memory and the current stream.
The binding raises if the shared library is missing or a call fails; there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsv4kv.so")

BF16, FP8_E4M3_ROW, FP4_E2M1_G16, FP8_E4M3_ROW_ROPE_BF16 = 0, 1, 2, 3
DEV_BAD_INDEX, DEV_TIMEOUT, DEV_INCONSISTENT, DEV_BAD_POOL = 0x1, 0x2, 0x4, 0x8
DEV_BAD_PAGE, DEV_BAD_LENGTH = 0x10, 0x20
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_WORKSPACE", 4: "ERR_CUDA"}


class Dsv4kvError(RuntimeError):
    def __init__(self, status: int, where: str, text: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {text}")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("dim", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class PagedDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("dim", ctypes.c_int32), ("page_rows", ctypes.c_int32),
                ("table_stride", ctypes.c_int32), ("pool_pages", ctypes.c_int64), ("table", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib: Optional[ctypes.CDLL] = None

_c = ctypes
_SIGS = {
    "dsv4kv_last_error": (_c.c_char_p, []),
    "dsv4kv_version": (_c.c_char_p, []),
    "dsv4kv_compress_entries": (_c.c_int64, [_c.c_int64, _c.c_int32, _c.c_int32]),
    "dsv4kv_compress": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int64, _c.c_int32, _c.c_int32,
                                   _c.c_int32, _c.c_int32, _c.c_int64, _c.c_int32, _c.c_double, _c.c_int32,
                                   _c.c_void_p, _c.c_void_p]),
    "dsv4kv_quantize": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.c_int64, _c.c_int32, _c.c_int32, _c.c_void_p,
                                   _c.c_void_p, _c.c_void_p]),
    "dsv4kv_index_topk_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int64, _c.c_int32]),
    "dsv4kv_index_topk": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.c_int32, _c.c_int64, _c.c_int32,
                                     _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "dsv4kv_index_score": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.c_int32, _c.c_int64, _c.c_int32,
                                      _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "dsv4kv_append": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_int64, _c.c_int32, _c.c_int32,
                                 _c.c_int32, _c.c_int32, _c.c_int32, _c.c_double, _c.c_void_p, _c.c_void_p,
                                 _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "dsv4kv_index_topk_pool_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32]),
    "dsv4kv_index_topk_pool": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.c_int32, _c.c_int64, _c.c_void_p,
                                          _c.c_int32, _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                          _c.c_size_t, _c.c_void_p]),
    "dsv4kv_index_select": (_c.c_int, [_c.c_int32, _c.c_int64, _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                       _c.c_size_t, _c.c_void_p]),
    "dsv4kv_index_topk_noalloc_max_scratch_bytes": (_c.c_size_t, []),
    "dsv4kv_index_topk_noalloc": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.c_int32, _c.c_int64, _c.c_int32,
                                             _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "dsv4kv_index_topk_noalloc_status": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.c_void_p]),
    "dsv4kv_selftest_wait_timeout": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "dsv4kv_sparse_decode_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int32,
                                                           _c.c_int32]),
    "dsv4kv_sparse_decode": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.POINTER(CacheDesc), _c.c_void_p,
                                        _c.c_int32, _c.c_int32, _c.c_int64, _c.c_int32, _c.c_int32, _c.c_int64,
                                        _c.c_float, _c.c_int32, _c.c_double, _c.c_int32, _c.c_void_p,
                                        _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "dsv4kv_index_topk_paged_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int64, _c.c_int32, _c.c_int32,
                                                              _c.c_int32]),
    "dsv4kv_index_topk_paged": (_c.c_int, [_c.c_void_p, _c.POINTER(PagedDesc), _c.c_int32, _c.c_void_p, _c.c_int64,
                                           _c.c_int32, _c.c_int32, _c.c_int32, _c.c_void_p, _c.c_void_p,
                                           _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "dsv4kv_sparse_decode_paged_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int32,
                                                                 _c.c_int32]),
    "dsv4kv_sparse_decode_paged": (_c.c_int, [_c.c_void_p, _c.POINTER(PagedDesc), _c.POINTER(PagedDesc),
                                              _c.c_void_p, _c.c_int32, _c.c_int32, _c.c_void_p, _c.c_int64,
                                              _c.c_int32, _c.c_int32, _c.c_int32, _c.c_float, _c.c_int32,
                                              _c.c_double, _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                              _c.c_void_p]),
    "dsv4kv_dense_decode_paged_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int64,
                                                                _c.c_int32, _c.c_int32]),
    "dsv4kv_dense_decode_paged": (_c.c_int, [_c.c_void_p, _c.POINTER(PagedDesc), _c.POINTER(PagedDesc), _c.c_int32,
                                             _c.c_int32, _c.c_void_p, _c.c_int64, _c.c_int32, _c.c_int32,
                                             _c.c_float, _c.c_int32, _c.c_double, _c.c_int32, _c.c_void_p,
                                             _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "dsv4kv_dense_decode_workspace_bytes": (_c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int64,
                                                          _c.c_int32]),
    "dsv4kv_dense_decode": (_c.c_int, [_c.c_void_p, _c.POINTER(CacheDesc), _c.POINTER(CacheDesc), _c.c_int32,
                                       _c.c_int32, _c.c_int64, _c.c_int32, _c.c_int64, _c.c_float, _c.c_int32,
                                       _c.c_double, _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                       _c.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """Load libdsv4kv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m compressed_sparse_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise Dsv4kvError(status, where, lib().dsv4kv_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


@dataclass
class Cache:
    """A cache tensor [B][rows][dim] in one of the three formats."""
    fmt: int
    codes: torch.Tensor                      # bf16/u16 [B][rows][dim], u8 [B][rows][dim] or [B][rows][dim/2]
    scales: Optional[torch.Tensor] = None    # None, f32 [B][rows], u8 [B][rows][dim/16]
    dim: int = 512

    @property
    def rows(self) -> int:
        return int(self.codes.shape[1]) if self.codes.dim() >= 2 else 0

    def desc(self) -> CacheDesc:
        return CacheDesc(self.fmt, self.dim, self.rows, _ptr(self.codes), _ptr(self.scales))


@dataclass
class PagedCache:
    """A paged cache: rows of every sequence in pages of `page_rows` rows of one shared pool.
    Row i of sequence b is pool row table[b][i // page_rows] * page_rows + i % page_rows."""
    fmt: int
    codes: torch.Tensor                      # pool rows: [pool_pages * page_rows][row bytes or channels]
    table: torch.Tensor                      # int32 [B][table_stride] page numbers
    page_rows: int
    scales: Optional[torch.Tensor] = None    # pool scales per row (fp8: f32 [rows], fp4: u8 [rows][dim/16])
    dim: int = 512

    @property
    def pool_pages(self) -> int:
        return int(self.codes.shape[0]) // self.page_rows

    def desc(self) -> PagedDesc:
        return PagedDesc(self.fmt, self.dim, self.page_rows, int(self.table.shape[1]), self.pool_pages,
                         _ptr(self.table), _ptr(self.codes), _ptr(self.scales))


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zero-filled workspace (the library leaves it zeroed after each call)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device or "cuda")


def workspace_status(ws: torch.Tensor) -> int:
    """The sticky device status word of a workspace (DEV_* flags)."""
    return int(ws[:4].view(torch.int32).item())


def compress_entries(t: int, window: int, stride: int) -> int:
    return int(lib().dsv4kv_compress_entries(t, window, stride))


def compress(s_raw: torch.Tensor, w: torch.Tensor, stride: int, window: int, pos0: int = 0, rope_dim: int = 64,
             rope_base: float = 10000.0, out_fp32: bool = False, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """s_raw bf16 [B][t][D], w f32 [K][D] -> entries [B][N][D] (bf16 or f32)."""
    b, t, d = s_raw.shape
    n = compress_entries(t, window, stride)
    if out is None:
        out = torch.empty((b, n, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=s_raw.device)
    _check(lib().dsv4kv_compress(_ptr(s_raw), _ptr(w), b, t, d, int(w.shape[0]), stride, window, pos0, rope_dim,
                                 rope_base, int(out_fp32), _ptr(out), _stream(stream)), "dsv4kv_compress")
    return out


def append(s_new: torch.Tensor, w: torch.Tensor, t: int, stride: int, window: int, raw_ring: torch.Tensor,
           win_ring: Optional[torch.Tensor], comp: torch.Tensor, rope_dim: int = 64, rope_base: float = 10000.0,
           stream=None) -> None:
    """Append the states s_new bf16 [B][D] of position t: raw ring [B][W+K][D], window ring [B][W][D] and,
    when an entry's block leaves the window, that entry into comp [B][rows][D] (all bf16)."""
    b, d = int(s_new.shape[0]), int(s_new.shape[1])
    _check(lib().dsv4kv_append(_ptr(s_new), _ptr(w), b, t, d, int(w.shape[0]), stride, window, rope_dim, rope_base,
                               _ptr(raw_ring), _ptr(win_ring) if win_ring is not None else None, _ptr(comp),
                               int(comp.shape[1]), _stream(stream)), "dsv4kv_append")


def quantize(x: torch.Tensor, fmt: int, codes: Optional[torch.Tensor] = None,
             scales: Optional[torch.Tensor] = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Rows x [..., D] (bf16 or f32) -> (codes, scales) in a quantised cache format: fp8 rows
    (codes [..., D], scales f32 [...]), fp4 (codes [..., D/2], E4M3 scales [..., D/16]) or fp8
    with the last 64 channels in bf16 (row bytes [..., D + 64], scales f32 [...])."""
    d = int(x.shape[-1])
    rows = x.numel() // d
    lead = tuple(x.shape[:-1])
    row_bytes = {FP8_E4M3_ROW: d, FP4_E2M1_G16: d // 2, FP8_E4M3_ROW_ROPE_BF16: d + 64}.get(fmt, d)
    if codes is None:
        codes = torch.empty(lead + (row_bytes,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = (torch.empty(lead + (d // 16,), dtype=torch.uint8, device=x.device) if fmt == FP4_E2M1_G16
                  else torch.empty(lead, dtype=torch.float32, device=x.device))
    _check(lib().dsv4kv_quantize(_ptr(x), int(x.dtype == torch.float32), rows, d, fmt, _ptr(codes), _ptr(scales),
                                 _stream(stream)), "dsv4kv_quantize")
    return codes, scales


def index_topk_workspace_bytes(batch: int, n: int, k: int) -> int:
    return int(lib().dsv4kv_index_topk_workspace_bytes(batch, n, k))


def index_topk(qidx: torch.Tensor, keys: Cache, n: int, k: int, idx_out: Optional[torch.Tensor] = None,
               count_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """qidx bf16 [B][128], keys [B][>=n][128] -> (idx int32 [B][k] ascending, -1 padded; count int32 [B])."""
    b = int(qidx.shape[0])
    dev = qidx.device
    if idx_out is None:
        idx_out = torch.empty((b, k), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((b,), dtype=torch.int32, device=dev)
    if ws is None:
        ws = new_workspace(index_topk_workspace_bytes(b, n, k), dev)
    d = keys.desc()
    _check(lib().dsv4kv_index_topk(_ptr(qidx), ctypes.byref(d), b, n, k, _ptr(idx_out), _ptr(count_out), _ptr(ws),
                                   ws.numel(), _stream(stream)), "dsv4kv_index_topk")
    return idx_out, count_out


def index_score(qidx: torch.Tensor, keys: Cache, n: int, k: int, ws: torch.Tensor, stream=None) -> None:
    """The scoring half of index_topk: scores and histogram into ws (index_topk_workspace_bytes sized)."""
    d = keys.desc()
    _check(lib().dsv4kv_index_score(_ptr(qidx), ctypes.byref(d), int(qidx.shape[0]), n, k, _ptr(ws), ws.numel(),
                                    _stream(stream)), "dsv4kv_index_score")


def index_select(batch: int, n: int, k: int, idx_out: torch.Tensor, count_out: Optional[torch.Tensor],
                 ws: torch.Tensor, stream=None) -> tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The selection half of index_topk, from the workspace index_score filled."""
    _check(lib().dsv4kv_index_select(batch, n, k, _ptr(idx_out), _ptr(count_out) if count_out is not None else None,
                                     _ptr(ws), ws.numel(), _stream(stream)), "dsv4kv_index_select")
    return idx_out, count_out


def index_topk_pool(qidx: torch.Tensor, keys: Cache, n: int, pool: torch.Tensor, k: int,
                    idx_out: Optional[torch.Tensor] = None, count_out: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k re-index inside a candidate pool: pool int32 [B][P] (ascending entries, negative = none)
    -> (idx int32 [B][k] ascending, -1 padded; count int32 [B])."""
    b = int(qidx.shape[0])
    p = int(pool.shape[1]) if pool.dim() == 2 else 0
    if idx_out is None:
        idx_out = torch.empty((b, k), dtype=torch.int32, device=qidx.device)
    if count_out is None:
        count_out = torch.empty((b,), dtype=torch.int32, device=qidx.device)
    if ws is None:
        ws = new_workspace(int(lib().dsv4kv_index_topk_pool_workspace_bytes(b, p, k)), qidx.device)
    d = keys.desc()
    _check(lib().dsv4kv_index_topk_pool(_ptr(qidx), ctypes.byref(d), b, n, _ptr(pool), p, k, _ptr(idx_out),
                                        _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)),
           "dsv4kv_index_topk_pool")
    return idx_out, count_out


def index_topk_noalloc(qidx: torch.Tensor, keys: Cache, n: int, k: int, idx_out: Optional[torch.Tensor] = None,
                       count_out: Optional[torch.Tensor] = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """index_topk with the library's static device scratch instead of a workspace (for callers that
    cannot allocate device memory; concurrent calls on the GPU race)."""
    b = int(qidx.shape[0])
    if idx_out is None:
        idx_out = torch.empty((b, k), dtype=torch.int32, device=qidx.device)
    if count_out is None:
        count_out = torch.empty((b,), dtype=torch.int32, device=qidx.device)
    d = keys.desc()
    _check(lib().dsv4kv_index_topk_noalloc(_ptr(qidx), ctypes.byref(d), b, n, k, _ptr(idx_out), _ptr(count_out),
                                           _stream(stream)), "dsv4kv_index_topk_noalloc")
    return idx_out, count_out


def index_topk_noalloc_status(clear: bool = False, stream=None) -> int:
    """The device status word (DEV_* flags) that the calls of index_topk_noalloc have accumulated in the
    static scratch since it was last cleared; `clear` zeroes it after reading."""
    word = torch.zeros(1, dtype=torch.int32).pin_memory()
    s = torch.cuda.current_stream() if stream is None else stream
    _check(lib().dsv4kv_index_topk_noalloc_status(_ptr(word), int(clear), _stream(s)),
           "dsv4kv_index_topk_noalloc_status")
    s.synchronize()
    return int(word.item()) & 0xffffffff


def selftest_wait_timeout(status: torch.Tensor, stream=None) -> None:
    """Launch the library's bounded-wait self-test: after about one second on the GPU it ORs DEV_TIMEOUT
    into `status` (one int32 on the device)."""
    _check(lib().dsv4kv_selftest_wait_timeout(_ptr(status), _stream(stream)), "dsv4kv_selftest_wait_timeout")


def sparse_decode_workspace_bytes(batch: int, heads: int, k: int, window: int, dim: int = 512) -> int:
    return int(lib().dsv4kv_sparse_decode_workspace_bytes(batch, heads, dim, k, window))


def dense_decode_workspace_bytes(batch: int, heads: int, n: int, window: int, dim: int = 512) -> int:
    return int(lib().dsv4kv_dense_decode_workspace_bytes(batch, heads, dim, n, window))


def sparse_decode(q: torch.Tensor, comp: Cache, win: Cache, idx: torch.Tensor, n: int, window: int, t: int,
                  sm_scale: Optional[float] = None, rope_dim: int = 64, rope_base: float = 10000.0,
                  out_fp32: bool = False, out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """q bf16 [B][H][512] -> out [B][H][512]; idx int32 [B][k] from index_topk."""
    b, h, d = q.shape
    k = int(idx.shape[1])
    if sm_scale is None:
        sm_scale = d ** -0.5
    if out is None:
        out = torch.empty((b, h, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    if ws is None:
        ws = new_workspace(sparse_decode_workspace_bytes(b, h, k, window, d), q.device)
    cd, wd = comp.desc(), win.desc()
    _check(lib().dsv4kv_sparse_decode(_ptr(q), ctypes.byref(cd), ctypes.byref(wd), _ptr(idx), b, h, n, window, k, t,
                                      sm_scale, rope_dim, rope_base, int(out_fp32), _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(stream)), "dsv4kv_sparse_decode")
    return out


def dense_decode(q: torch.Tensor, comp: Cache, win: Cache, n: int, window: int, t: int,
                 sm_scale: Optional[float] = None, rope_dim: int = 64, rope_base: float = 10000.0,
                 out_fp32: bool = False, out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """q bf16 [B][H][512] -> out [B][H][512] over all n compressed rows plus the window."""
    b, h, d = q.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    if out is None:
        out = torch.empty((b, h, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    if ws is None:
        ws = new_workspace(dense_decode_workspace_bytes(b, h, n, window, d), q.device)
    cd, wd = comp.desc(), win.desc()
    _check(lib().dsv4kv_dense_decode(_ptr(q), ctypes.byref(cd), ctypes.byref(wd), b, h, n, window, t, sm_scale,
                                     rope_dim, rope_base, int(out_fp32), _ptr(out), _ptr(ws), ws.numel(),
                                     _stream(stream)), "dsv4kv_dense_decode")
    return out


def index_topk_paged(qidx: torch.Tensor, keys: PagedCache, t_seq: torch.Tensor, t_max: int, k: int,
                     window: int = 128, stride: int = 4, idx_out: Optional[torch.Tensor] = None,
                     count_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Ragged, paged top-k: t_seq int64 [B] (device) query positions, sequence b has
    max(0, (t_b - window) // stride) keys -> (idx int32 [B][k] ascending, -1 padded; count int32 [B])."""
    b = int(qidx.shape[0])
    dev = qidx.device
    if idx_out is None:
        idx_out = torch.empty((b, k), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((b,), dtype=torch.int32, device=dev)
    if ws is None:
        ws = new_workspace(int(lib().dsv4kv_index_topk_paged_workspace_bytes(b, t_max, window, stride, k)), dev)
    d = keys.desc()
    _check(lib().dsv4kv_index_topk_paged(_ptr(qidx), ctypes.byref(d), b, _ptr(t_seq), t_max, window, stride, k,
                                         _ptr(idx_out), _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)),
           "dsv4kv_index_topk_paged")
    return idx_out, count_out


def sparse_decode_paged(q: torch.Tensor, comp: PagedCache, win: PagedCache, idx: torch.Tensor, t_seq: torch.Tensor,
                        t_max: int, window: int = 128, stride: int = 4, sm_scale: Optional[float] = None,
                        rope_dim: int = 64, rope_base: float = 10000.0, out_fp32: bool = False,
                        out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """Ragged, paged c4a decode: q bf16 [B][H][512], idx int32 [B][k] from index_topk_paged."""
    b, h, d = q.shape
    k = int(idx.shape[1])
    if sm_scale is None:
        sm_scale = d ** -0.5
    if out is None:
        out = torch.empty((b, h, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    if ws is None:
        ws = new_workspace(int(lib().dsv4kv_sparse_decode_paged_workspace_bytes(b, h, d, k, window)), q.device)
    cd, wd = comp.desc(), win.desc()
    _check(lib().dsv4kv_sparse_decode_paged(_ptr(q), ctypes.byref(cd), ctypes.byref(wd), _ptr(idx), b, h, _ptr(t_seq),
                                            t_max, window, stride, k, sm_scale, rope_dim, rope_base, int(out_fp32),
                                            _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "dsv4kv_sparse_decode_paged")
    return out


def dense_decode_paged(q: torch.Tensor, comp: PagedCache, win: PagedCache, t_seq: torch.Tensor, t_max: int,
                       window: int = 128, stride: int = 128, sm_scale: Optional[float] = None, rope_dim: int = 64,
                       rope_base: float = 10000.0, out_fp32: bool = False, out: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Ragged, paged c128a decode over every sequence's n_b entries plus its window rows."""
    b, h, d = q.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    if out is None:
        out = torch.empty((b, h, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    if ws is None:
        ws = new_workspace(int(lib().dsv4kv_dense_decode_paged_workspace_bytes(b, h, d, t_max, window, stride)),
                           q.device)
    cd, wd = comp.desc(), win.desc()
    _check(lib().dsv4kv_dense_decode_paged(_ptr(q), ctypes.byref(cd), ctypes.byref(wd), b, h, _ptr(t_seq), t_max,
                                           window, stride, sm_scale, rope_dim, rope_base, int(out_fp32), _ptr(out),
                                           _ptr(ws), ws.numel(), _stream(stream)), "dsv4kv_dense_decode_paged")
    return out
