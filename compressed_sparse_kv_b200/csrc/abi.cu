// Exported C ABI of libdsv4kv: argument validation, workspace sizing and
// kernel launches on the caller's stream.  No allocation, no host sync.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

#define DSV4KV_API extern "C" __attribute__((visibility("default")))

namespace dsv4kv {

static thread_local char g_err[512] = "";

dsv4kv_status set_error(dsv4kv_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

dsv4kv_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSV4KV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return DSV4KV_OK;
}

int sm_count() {
  static std::atomic<int> cache[64];  // per device; 0 = not queried yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                    CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_nd(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(map, dtype, cuuint32_t(rank), const_cast<void*>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static dsv4kv_status check_cache(const dsv4kv_cache* c, const char* what, int64_t need_rows, int dim) {
  if (!c) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: cache descriptor is null", what);
  if (c->dim != dim) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: dim %d, expected %d", what, c->dim, dim);
  if (c->rows < need_rows)
    return set_error(DSV4KV_ERR_INVALID_ARG, "%s: %lld rows per sequence < %lld needed", what, (long long)c->rows,
                     (long long)need_rows);
  if (need_rows == 0) return DSV4KV_OK;
  if (!c->codes || !aligned16(c->codes))
    return set_error(DSV4KV_ERR_INVALID_ARG, "%s: codes pointer null or not 16-byte aligned", what);
  if (c->fmt == DSV4KV_BF16) return DSV4KV_OK;
  if (c->fmt == DSV4KV_FP8_E4M3_ROW || c->fmt == DSV4KV_FP4_E2M1_G16 || c->fmt == DSV4KV_FP8_E4M3_ROW_ROPE_BF16) {
    if (!c->scales || !aligned16(c->scales))
      return set_error(DSV4KV_ERR_INVALID_ARG, "%s: scales pointer null or not 16-byte aligned", what);
    return DSV4KV_OK;
  }
  return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: unknown format %d", what, c->fmt);
}

}  // namespace dsv4kv

using namespace dsv4kv;

DSV4KV_API const char* dsv4kv_last_error(void) { return g_err; }

DSV4KV_API const char* dsv4kv_version(void) { return "dsv4kv 0.1 (sm_100a)"; }

DSV4KV_API dsv4kv_status dsv4kv_selftest_wait_timeout(uint32_t* status, void* stream) {
  if (!status) return set_error(DSV4KV_ERR_INVALID_ARG, "selftest_wait_timeout: status is null");
  return selftest_wait_timeout_launch(status, static_cast<cudaStream_t>(stream));
}

DSV4KV_API int64_t dsv4kv_compress_entries(int64_t t, int32_t window, int32_t stride) {
  if (stride <= 0 || t < window) return 0;
  return (t - window) / stride;
}

DSV4KV_API dsv4kv_status dsv4kv_compress(const void* s_raw, const float* w, int32_t batch, int64_t t, int32_t dim,
                                         int32_t k_taps, int32_t stride, int32_t window, int64_t pos0,
                                         int32_t rope_dim, double rope_base, int32_t out_fp32, void* out,
                                         void* stream) {
  g_err[0] = 0;
  if (batch < 0 || t < 0 || k_taps < 1 || stride < 1 || window < 0)
    return set_error(DSV4KV_ERR_INVALID_ARG, "compress: bad sizes");
  if (rope_dim < 0 || rope_dim > dim || (rope_dim & 1))
    return set_error(DSV4KV_ERR_INVALID_ARG, "compress: rope_dim must be even and <= dim");
  if (!(rope_base > 0.0)) return set_error(DSV4KV_ERR_INVALID_ARG, "compress: rope_base must be > 0");
  const int64_t n = dsv4kv_compress_entries(t, window, stride);
  if (batch == 0 || n == 0) return DSV4KV_OK;
  if (!s_raw || !w || !out || !aligned16(s_raw) || !aligned16(w) || !aligned16(out))
    return set_error(DSV4KV_ERR_INVALID_ARG, "compress: null or misaligned pointer");
  return compress_launch(s_raw, w, batch, t, dim, k_taps, stride, window, pos0, rope_dim, rope_base, out_fp32, out,
                         static_cast<cudaStream_t>(stream));
}

DSV4KV_API dsv4kv_status dsv4kv_append(const void* s_new, const float* w, int32_t batch, int64_t t, int32_t dim,
                                       int32_t k_taps, int32_t stride, int32_t window, int32_t rope_dim,
                                       double rope_base, void* raw_ring, void* win_ring, void* comp,
                                       int64_t comp_rows, void* stream) {
  g_err[0] = 0;
  if (batch < 0 || t < 0 || k_taps < 1 || stride < 1 || window < 0 || comp_rows < 0)
    return set_error(DSV4KV_ERR_INVALID_ARG, "append: bad sizes");
  if (rope_dim < 0 || rope_dim > dim || (rope_dim & 1))
    return set_error(DSV4KV_ERR_INVALID_ARG, "append: rope_dim must be even and <= dim");
  if (!(rope_base > 0.0)) return set_error(DSV4KV_ERR_INVALID_ARG, "append: rope_base must be > 0");
  if (batch == 0) return DSV4KV_OK;
  if (!s_new || !w || !raw_ring || !aligned16(s_new) || !aligned16(w) || !aligned16(raw_ring))
    return set_error(DSV4KV_ERR_INVALID_ARG, "append: null or misaligned pointer");
  if (window > 0 && (!win_ring || !aligned16(win_ring)))
    return set_error(DSV4KV_ERR_INVALID_ARG, "append: window ring null or misaligned");
  const int64_t emit = append_emit_entry(t, window, stride);
  if (emit >= 0 && (!comp || !aligned16(comp) || emit >= comp_rows))
    return set_error(DSV4KV_ERR_INVALID_ARG, "append: entry %lld does not fit the compressed cache", (long long)emit);
  return append_launch(s_new, w, batch, t, dim, k_taps, stride, window, rope_dim, rope_base, raw_ring, win_ring, comp,
                       comp_rows, static_cast<cudaStream_t>(stream));
}

DSV4KV_API dsv4kv_status dsv4kv_quantize(const void* in, int32_t in_fp32, int64_t rows, int32_t dim, int32_t fmt,
                                         void* codes, void* scales, void* stream) {
  g_err[0] = 0;
  if (rows < 0) return set_error(DSV4KV_ERR_INVALID_ARG, "quantize: rows < 0");
  if (fmt != DSV4KV_FP8_E4M3_ROW && fmt != DSV4KV_FP4_E2M1_G16 && fmt != DSV4KV_FP8_E4M3_ROW_ROPE_BF16)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "quantize: format %d is not a quantised format", fmt);
  if (rows == 0) return DSV4KV_OK;
  if (!in || !codes || !scales || !aligned16(in) || !aligned16(codes) || !aligned16(scales))
    return set_error(DSV4KV_ERR_INVALID_ARG, "quantize: null or misaligned pointer");
  return quantize_launch(in, in_fp32, rows, dim, fmt, codes, scales, static_cast<cudaStream_t>(stream));
}

DSV4KV_API size_t dsv4kv_index_topk_workspace_bytes(int32_t batch, int64_t n, int32_t k) {
  if (batch < 0 || n < 0 || k < 1) return 0;
  return index_topk_ws_bytes(batch, n, k);
}

// Shared checks of the indexer calls (what = the call's name for messages).
static dsv4kv_status check_index(const char* what, const void* qidx, const dsv4kv_cache* keys, int32_t batch,
                                 int64_t n, int32_t k, bool need_keys, bool need_out, const int32_t* idx_out,
                                 const void* ws, size_t ws_bytes) {
  if (batch < 0 || n < 0) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: bad sizes", what);
  if (k < 1 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: k must be in [1, 2048]", what);
  if (batch == 0) return DSV4KV_OK;
  if (need_out && !idx_out) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: idx_out is null", what);
  if (need_keys) {
    if (!keys) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: keys is null", what);
    if (keys->fmt != DSV4KV_BF16 && keys->fmt != DSV4KV_FP4_E2M1_G16)
      return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: keys must be bf16 or fp4", what);
    dsv4kv_status st = check_cache(keys, what, n, 128);
    if (st != DSV4KV_OK) return st;
    if (n > k && (!qidx || !aligned16(qidx))) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: qidx null or misaligned", what);
  }
  if (n > k) {
    if (int64_t(batch) * n > (int64_t(1) << 40)) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: too large", what);
    if (!ws || ws_bytes < index_topk_ws_bytes(batch, n, k))
      return set_error(DSV4KV_ERR_WORKSPACE, "%s: workspace null or too small", what);
  }
  return DSV4KV_OK;
}

DSV4KV_API dsv4kv_status dsv4kv_index_topk(const void* qidx, const dsv4kv_cache* keys, int32_t batch, int64_t n,
                                           int32_t k, int32_t* idx_out, int32_t* count_out, void* ws,
                                           size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  dsv4kv_status st = check_index("index_topk", qidx, keys, batch, n, k, true, true, idx_out, ws, ws_bytes);
  if (st != DSV4KV_OK || batch == 0) return st;
  return index_topk_launch(static_cast<const uint16_t*>(qidx), *keys, batch, n, k, idx_out, count_out, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

DSV4KV_API dsv4kv_status dsv4kv_index_score(const void* qidx, const dsv4kv_cache* keys, int32_t batch, int64_t n,
                                            int32_t k, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  dsv4kv_status st = check_index("index_score", qidx, keys, batch, n, k, true, false, nullptr, ws, ws_bytes);
  if (st != DSV4KV_OK || batch == 0) return st;
  return index_score_launch(static_cast<const uint16_t*>(qidx), *keys, batch, n, k, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));
}

DSV4KV_API dsv4kv_status dsv4kv_index_select(int32_t batch, int64_t n, int32_t k, int32_t* idx_out,
                                             int32_t* count_out, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  dsv4kv_status st = check_index("index_select", nullptr, nullptr, batch, n, k, false, true, idx_out, ws, ws_bytes);
  if (st != DSV4KV_OK || batch == 0) return st;
  return index_select_launch(batch, n, k, idx_out, count_out, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

DSV4KV_API size_t dsv4kv_index_topk_pool_workspace_bytes(int32_t batch, int32_t pool_cap, int32_t k) {
  if (batch < 0 || pool_cap < 0 || k < 1) return 0;
  return 16;  // the status word
}

DSV4KV_API dsv4kv_status dsv4kv_index_topk_pool(const void* qidx, const dsv4kv_cache* keys, int32_t batch, int64_t n,
                                                const int32_t* pool, int32_t pool_cap, int32_t k, int32_t* idx_out,
                                                int32_t* count_out, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  if (batch < 0 || n < 0 || pool_cap < 0) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_pool: bad sizes");
  if (k < 1 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_pool: k must be in [1, 2048]");
  if (pool_cap > 8192) return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_pool: pool_cap must be <= 8192");
  if (batch == 0) return DSV4KV_OK;
  if (!idx_out) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_pool: idx_out is null");
  if (pool_cap > 0 && !pool) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_pool: pool is null");
  if (!keys) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_pool: keys is null");
  if (keys->fmt != DSV4KV_BF16 && keys->fmt != DSV4KV_FP4_E2M1_G16)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_pool: keys must be bf16 or fp4");
  dsv4kv_status st = check_cache(keys, "index_topk_pool", n, 128);
  if (st != DSV4KV_OK) return st;
  if (!qidx || !aligned16(qidx)) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_pool: qidx null or misaligned");
  if (!ws || ws_bytes < 16) return set_error(DSV4KV_ERR_WORKSPACE, "index_topk_pool: workspace null or too small");
  return index_topk_pool_launch(static_cast<const uint16_t*>(qidx), *keys, batch, n, pool, pool_cap, k, idx_out,
                                count_out, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

static dsv4kv_status check_decode(const void* q, const dsv4kv_cache* comp, const dsv4kv_cache* win, int32_t batch,
                                  int32_t heads, int64_t n, int32_t window, int64_t need_comp_rows, const void* out) {
  if (batch < 1) return set_error(DSV4KV_ERR_INVALID_ARG, "decode: batch must be >= 1");
  if (heads < 1 || heads > 64) return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: heads must be in [1, 64]");
  if (n < 0 || window < 0) return set_error(DSV4KV_ERR_INVALID_ARG, "decode: negative sizes");
  if (!q || !aligned16(q) || !out || !aligned16(out))
    return set_error(DSV4KV_ERR_INVALID_ARG, "decode: q/out null or misaligned");
  if (!comp || !win) return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cache descriptor is null");
  dsv4kv_status st = check_cache(comp, "decode comp", need_comp_rows, 512);
  if (st != DSV4KV_OK) return st;
  st = check_cache(win, "decode window", window, 512);
  if (st != DSV4KV_OK) return st;
  if (int64_t(batch) * std::max<int64_t>(comp->rows, 1) >= (int64_t(1) << 31) ||
      int64_t(batch) * std::max<int64_t>(win->rows, 1) >= (int64_t(1) << 31))
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: batch x rows must be < 2^31");
  return DSV4KV_OK;
}

DSV4KV_API size_t dsv4kv_sparse_decode_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int32_t k,
                                                       int32_t window) {
  if (batch < 1 || heads < 1 || k < 0 || window < 0) return 0;
  return decode_ws_bytes(batch, heads, dim, int64_t(k) + window);
}

DSV4KV_API size_t dsv4kv_dense_decode_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int64_t n,
                                                      int32_t window) {
  if (batch < 1 || heads < 1 || n < 0 || window < 0) return 0;
  return decode_ws_bytes(batch, heads, dim, n + window);
}

DSV4KV_API dsv4kv_status dsv4kv_sparse_decode(const void* q, const dsv4kv_cache* comp, const dsv4kv_cache* win,
                                              const int32_t* idx, int32_t batch, int32_t heads, int64_t n,
                                              int32_t window, int32_t k, int64_t t, float sm_scale,
                                              int32_t rope_dim, double rope_base, int32_t out_fp32, void* out,
                                              void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  if (k < 0 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "sparse_decode: k must be in [0, 2048]");
  dsv4kv_status st = check_decode(q, comp, win, batch, heads, n, window, n, out);
  if (st != DSV4KV_OK) return st;
  if (k > 0 && n > 0 && !idx) return set_error(DSV4KV_ERR_INVALID_ARG, "sparse_decode: idx is null");
  if (rope_dim < 0 || rope_dim > 512 || (rope_dim & 1))
    return set_error(DSV4KV_ERR_INVALID_ARG, "sparse_decode: bad rope_dim");
  if (!ws || ws_bytes < dsv4kv_sparse_decode_workspace_bytes(batch, heads, 512, k, window))
    return set_error(DSV4KV_ERR_WORKSPACE, "sparse_decode: workspace null or too small");
  DecodeArgs a{q, *comp, *win, idx, batch, heads, 512, n, window, k, t, sm_scale, rope_dim, rope_base, out_fp32, out};
  return decode_launch(a, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ paged, ragged
// Checks a paged cache whose sequences have at most `max_rows` rows and
// turns it into the kernels' form (a pool "cache" of pool rows + its pages).
static dsv4kv_status check_paged(const dsv4kv_paged_cache* c, const char* what, int64_t max_rows, int dim,
                                 bool keys, dsv4kv_cache* pool, PageDesc* pg) {
  if (!c) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: paged cache descriptor is null", what);
  if (c->dim != dim) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: dim %d, expected %d", what, c->dim, dim);
  if (keys ? (c->fmt != DSV4KV_BF16 && c->fmt != DSV4KV_FP4_E2M1_G16)
           : (c->fmt < DSV4KV_BF16 || c->fmt > DSV4KV_FP8_E4M3_ROW_ROPE_BF16))
    return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: format %d", what, c->fmt);
  if (c->page_rows <= 0 || c->page_rows % 64 != 0)
    return set_error(DSV4KV_ERR_INVALID_ARG, "%s: page_rows must be a positive multiple of 64", what);
  if (c->pool_pages < 1 || c->pool_pages * int64_t(c->page_rows) >= (int64_t(1) << 31))
    return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: the pool must hold between 1 page and 2^31 rows", what);
  const int64_t need_pages = (max_rows + c->page_rows - 1) / c->page_rows;
  if (c->table_stride < need_pages)
    return set_error(DSV4KV_ERR_INVALID_ARG, "%s: table_stride %d < %lld pages a sequence may need", what,
                     c->table_stride, (long long)need_pages);
  if (max_rows > 0 && !c->table) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: block table is null", what);
  dsv4kv_cache d{c->fmt, c->dim, c->pool_pages * int64_t(c->page_rows), c->codes, c->scales};
  dsv4kv_status st = check_cache(&d, what, max_rows > 0 ? 1 : 0, dim);
  if (st != DSV4KV_OK) return st;
  *pool = d;
  *pg = PageDesc{c->table, c->page_rows, c->table_stride, c->pool_pages};
  return DSV4KV_OK;
}

static dsv4kv_status check_ragged(const char* what, int32_t batch, const int64_t* t_seq, int64_t t_max,
                                  int32_t window, int32_t stride) {
  if (batch < 1) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: batch must be >= 1", what);
  if (!t_seq) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: t_seq is null", what);
  if (t_max < 0 || window < 0 || stride < 1) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: bad sizes", what);
  if (t_max >= (int64_t(1) << 40)) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: t_max too large", what);
  return DSV4KV_OK;
}

DSV4KV_API size_t dsv4kv_index_topk_paged_workspace_bytes(int32_t batch, int64_t t_max, int32_t window, int32_t stride,
                                                          int32_t k) {
  if (batch < 0 || t_max < 0 || window < 0 || stride < 1 || k < 1) return 0;
  return index_topk_ws_bytes(batch, dsv4kv_compress_entries(t_max, window, stride), k);
}

DSV4KV_API dsv4kv_status dsv4kv_index_topk_paged(const void* qidx, const dsv4kv_paged_cache* keys, int32_t batch,
                                                 const int64_t* t_seq, int64_t t_max, int32_t window, int32_t stride,
                                                 int32_t k, int32_t* idx_out, int32_t* count_out, void* ws,
                                                 size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  const char* what = "index_topk_paged";
  dsv4kv_status st = check_ragged(what, batch, t_seq, t_max, window, stride);
  if (st != DSV4KV_OK) return st;
  if (k < 1 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: k must be in [1, 2048]", what);
  if (!idx_out) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: idx_out is null", what);
  const int64_t n_max = dsv4kv_compress_entries(t_max, window, stride);
  dsv4kv_cache pool{};
  PageDesc pg{};
  st = check_paged(keys, what, n_max, 128, true, &pool, &pg);
  if (st != DSV4KV_OK) return st;
  if (n_max > k) {
    if (!qidx || !aligned16(qidx)) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: qidx null or misaligned", what);
    if (int64_t(batch) * n_max > (int64_t(1) << 40)) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: too large", what);
  }
  if (!ws || ws_bytes < dsv4kv_index_topk_paged_workspace_bytes(batch, t_max, window, stride, k))
    return set_error(DSV4KV_ERR_WORKSPACE, "%s: workspace null or too small", what);
  Ragged rg;
  rg.t_seq = t_seq;
  rg.t_max = t_max;
  rg.window = window;
  rg.stride = stride;
  return index_topk_paged_launch(static_cast<const uint16_t*>(qidx), pool, pg, batch, rg, k, idx_out, count_out, ws,
                                 ws_bytes, static_cast<cudaStream_t>(stream));
}

DSV4KV_API size_t dsv4kv_sparse_decode_paged_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int32_t k,
                                                             int32_t window) {
  return dsv4kv_sparse_decode_workspace_bytes(batch, heads, dim, k, window);
}

DSV4KV_API size_t dsv4kv_dense_decode_paged_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int64_t t_max,
                                                            int32_t window, int32_t stride) {
  if (stride < 1 || t_max < 0) return 0;
  return dsv4kv_dense_decode_workspace_bytes(batch, heads, dim, dsv4kv_compress_entries(t_max, window, stride),
                                             window);
}

static dsv4kv_status decode_paged(const char* what, const void* q, const dsv4kv_paged_cache* comp,
                                  const dsv4kv_paged_cache* win, const int32_t* idx, int32_t batch, int32_t heads,
                                  const int64_t* t_seq, int64_t t_max, int32_t window, int32_t stride, int32_t k,
                                  float sm_scale, int32_t rope_dim, double rope_base, int32_t out_fp32, void* out,
                                  void* ws, size_t ws_bytes, void* stream) {
  dsv4kv_status st = check_ragged(what, batch, t_seq, t_max, window, stride);
  if (st != DSV4KV_OK) return st;
  if (heads < 1 || heads > 64) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: heads must be in [1, 64]", what);
  if (!q || !aligned16(q) || !out || !aligned16(out))
    return set_error(DSV4KV_ERR_INVALID_ARG, "%s: q/out null or misaligned", what);
  if (rope_dim < 0 || rope_dim > 512 || (rope_dim & 1)) return set_error(DSV4KV_ERR_INVALID_ARG, "%s: bad rope_dim", what);
  const int64_t n_max = dsv4kv_compress_entries(t_max, window, stride);
  const int32_t w_max = int32_t(std::min<int64_t>(t_max, window));
  if (n_max > (int64_t(1) << 30)) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: too many entries", what);
  dsv4kv_cache cpool{}, wpool{};
  PageDesc cpg{}, wpg{};
  st = check_paged(comp, what, n_max, 512, false, &cpool, &cpg);
  if (st != DSV4KV_OK) return st;
  st = check_paged(win, what, w_max, 512, false, &wpool, &wpg);
  if (st != DSV4KV_OK) return st;
  if (win->fmt != comp->fmt)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: the window cache must have the compressed cache's format", what);
  if (idx) {
    if (k < 0 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "%s: k must be in [0, 2048]", what);
    if (!ws || ws_bytes < dsv4kv_sparse_decode_workspace_bytes(batch, heads, 512, k, window))
      return set_error(DSV4KV_ERR_WORKSPACE, "%s: workspace null or too small", what);
  } else if (!ws || ws_bytes < dsv4kv_dense_decode_workspace_bytes(batch, heads, 512, n_max, window)) {
    return set_error(DSV4KV_ERR_WORKSPACE, "%s: workspace null or too small", what);
  }
  DecodeArgs a{q, cpool, wpool, idx, batch, heads, 512, n_max, window, idx ? k : 0, t_max, sm_scale, rope_dim,
               rope_base, out_fp32, out};
  a.t_seq = t_seq;
  a.t_max = t_max;
  a.stride = stride;
  a.comp_pg = cpg;
  a.win_pg = wpg;
  return decode_launch(a, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

DSV4KV_API dsv4kv_status dsv4kv_sparse_decode_paged(const void* q, const dsv4kv_paged_cache* comp,
                                                    const dsv4kv_paged_cache* win, const int32_t* idx, int32_t batch,
                                                    int32_t heads, const int64_t* t_seq, int64_t t_max, int32_t window,
                                                    int32_t stride, int32_t k, float sm_scale, int32_t rope_dim,
                                                    double rope_base, int32_t out_fp32, void* out, void* ws,
                                                    size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  if (!idx) return set_error(DSV4KV_ERR_INVALID_ARG, "sparse_decode_paged: idx is null");
  return decode_paged("sparse_decode_paged", q, comp, win, idx, batch, heads, t_seq, t_max, window, stride, k,
                      sm_scale, rope_dim, rope_base, out_fp32, out, ws, ws_bytes, stream);
}

DSV4KV_API dsv4kv_status dsv4kv_dense_decode_paged(const void* q, const dsv4kv_paged_cache* comp,
                                                   const dsv4kv_paged_cache* win, int32_t batch, int32_t heads,
                                                   const int64_t* t_seq, int64_t t_max, int32_t window, int32_t stride,
                                                   float sm_scale, int32_t rope_dim, double rope_base,
                                                   int32_t out_fp32, void* out, void* ws, size_t ws_bytes,
                                                   void* stream) {
  g_err[0] = 0;
  return decode_paged("dense_decode_paged", q, comp, win, nullptr, batch, heads, t_seq, t_max, window, stride, 0,
                      sm_scale, rope_dim, rope_base, out_fp32, out, ws, ws_bytes, stream);
}

DSV4KV_API dsv4kv_status dsv4kv_dense_decode(const void* q, const dsv4kv_cache* comp, const dsv4kv_cache* win,
                                             int32_t batch, int32_t heads, int64_t n, int32_t window, int64_t t,
                                             float sm_scale, int32_t rope_dim, double rope_base, int32_t out_fp32,
                                             void* out, void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  dsv4kv_status st = check_decode(q, comp, win, batch, heads, n, window, n, out);
  if (st != DSV4KV_OK) return st;
  if (rope_dim < 0 || rope_dim > 512 || (rope_dim & 1))
    return set_error(DSV4KV_ERR_INVALID_ARG, "dense_decode: bad rope_dim");
  if (n > (int64_t(1) << 30)) return set_error(DSV4KV_ERR_UNSUPPORTED, "dense_decode: n too large");
  if (!ws || ws_bytes < dsv4kv_dense_decode_workspace_bytes(batch, heads, 512, n, window))
    return set_error(DSV4KV_ERR_WORKSPACE, "dense_decode: workspace null or too small");
  DecodeArgs a{q, *comp, *win, nullptr, batch, heads, 512, n, window, 0, t, sm_scale, rope_dim, rope_base, out_fp32, out};
  return decode_launch(a, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}
