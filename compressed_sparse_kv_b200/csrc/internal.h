// Host-side declarations shared by the dsv4kv translation units (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <utility>
#include <cstdint>

#include "dsv4kv.h"

namespace dsv4kv {

dsv4kv_status set_error(dsv4kv_status st, const char* fmt, ...);

// Launch with programmatic stream serialisation (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// Same, with thread-block clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, unsigned cluster,
                               cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
dsv4kv_status check_launch(const char* what);
dsv4kv_status selftest_wait_timeout_launch(uint32_t* status, cudaStream_t stream);
int sm_count();
// The current device (0 when it cannot be read or is >= 64).  One-time set-up
// of a kernel (shared-memory limits, occupancy queries) is kept per device,
// so a process that drives several GPUs sets every one of them up.
inline int current_device() {
  int d = 0;
  return (cudaGetDevice(&d) == cudaSuccess && d >= 0 && d < 64) ? d : 0;
}
inline bool done_on_device(const std::atomic<uint64_t>& mask) {
  return (mask.load(std::memory_order_acquire) >> current_device()) & 1u;
}
inline void mark_done_on_device(std::atomic<uint64_t>& mask) {
  mask.fetch_or(uint64_t(1) << current_device(), std::memory_order_acq_rel);
}

// Driver entry point for cuTensorMapEncodeTiled (resolved once through the runtime).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);
// rank <= 5; strides_bytes[i] is the stride of dimension i + 1.
bool encode_tmap_nd(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                    uint32_t b2, CUtensorMapSwizzle swizzle);

size_t index_topk_ws_bytes(int batch, int64_t n, int k);
size_t index_topk_zero_prefix_bytes(int batch);
dsv4kv_status index_score_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n, int k,
                                 void* ws, size_t ws_bytes, cudaStream_t stream);
int64_t append_emit_entry(int64_t t, int window, int stride);
dsv4kv_status append_launch(const void* s_new, const float* w, int batch, int64_t t, int dim, int k_taps, int stride,
                            int window, int rope_dim, double rope_base, void* raw_ring, void* win_ring, void* comp,
                            int64_t comp_rows, cudaStream_t stream);
// A ragged batch (t_seq null: every sequence has the call's n entries).
struct Ragged {
  const int64_t* t_seq = nullptr;
  int64_t t_max = 0;
  int window = 0, stride = 1;
};
// Pages of a paged cache (table null: the dense [B][rows] layout of a dsv4kv_cache).
struct PageDesc {
  const int32_t* table;
  int page_rows, table_stride;
  int64_t pool_pages;
};
dsv4kv_status index_select_launch(int batch, int64_t n, int k, int32_t* idx_out, int32_t* count_out, void* ws,
                                  size_t ws_bytes, cudaStream_t stream, const Ragged& rg = Ragged{});
dsv4kv_status index_topk_paged_launch(const uint16_t* qidx, const dsv4kv_cache& pool, const PageDesc& pg, int batch,
                                      const Ragged& rg, int k, int32_t* idx_out, int32_t* count_out, void* ws,
                                      size_t ws_bytes, cudaStream_t stream);
dsv4kv_status index_topk_pool_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n,
                                     const int32_t* pool, int pool_cap, int k, int32_t* idx_out, int32_t* count_out,
                                     void* ws, size_t ws_bytes, cudaStream_t stream);
dsv4kv_status index_topk_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n, int k,
                                int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                                cudaStream_t stream);

struct DecodeArgs {
  const void* q;
  dsv4kv_cache comp;   // paged: codes / scales are the pools, rows = pool rows
  dsv4kv_cache win;
  const int32_t* idx;  // null for dense
  int batch, heads, dim;
  int64_t n;           // uniform: entries; ragged: the most any sequence has
  int window;          // uniform: window rows; ragged: the window length W
  int k;               // sparse only
  int64_t t;
  float sm_scale;
  int rope_dim;
  double rope_base;
  int out_fp32;
  void* out;
  // ragged batch (t_seq null: uniform)
  const int64_t* t_seq = nullptr;
  int64_t t_max = 0;
  int stride = 1;
  PageDesc comp_pg{}, win_pg{};
};
size_t decode_ws_bytes(int batch, int heads, int dim, int64_t rows_per_seq);
dsv4kv_status decode_launch(const DecodeArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream);

dsv4kv_status compress_launch(const void* s_raw, const float* w, int batch, int64_t t, int dim, int k_taps,
                              int stride, int window, int64_t pos0, int rope_dim, double rope_base,
                              int out_fp32, void* out, cudaStream_t stream);

dsv4kv_status quantize_launch(const void* in, int in_fp32, int64_t rows, int dim, int fmt, void* codes,
                              void* scales, cudaStream_t stream);

}  // namespace dsv4kv
