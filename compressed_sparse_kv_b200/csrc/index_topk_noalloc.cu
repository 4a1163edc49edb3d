// dsv4kv_index_topk_noalloc: the indexer top-k with its scratch in a
// file-scope device array instead of a caller workspace.
//
// Some callers cannot allocate device memory for a workspace: for example a
// serving engine whose memory manager has already reserved nearly all of HBM
// for its KV block pool, a plugin host that forbids device allocations, or a
// latency-critical path that must not pay for cudaMalloc's implicit
// synchronisation.  They still pass the inputs and outputs; the scratch comes
// from `g_index_scratch` below, which every GPU that loads this library keeps
// until the process exits.
//
// Set-up: every call looks up the array's device address on the current
// device with cudaGetSymbolAddress (in host code the symbol is only a
// stand-in, never a device pointer).  The first lookup on a device loads the
// library's device code there, so make the first call before any stream
// capture.  Looking the address up on every call (it is cheap) keeps it right
// after a cudaDeviceReset.  Every call shares the array, so calls that overlap
// on the GPU (other streams, other threads) race.  The counters and histograms
// that must start at zero are cleared on the stream at the start of every
// call; the status word in front of them is not: it accumulates the device
// flags of every call until dsv4kv_index_topk_noalloc_status reads (and, if
// asked, clears) it.
#include <cstdio>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

// Maximum scratch: 8 MiB (fits, e.g., batch 32 x 32736 entries with k = 512).
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
// The status word occupies the first 16 bytes of the scratch (as of a workspace).
constexpr size_t kStatusBytes = 16;

static __device__ __align__(256) unsigned char g_index_scratch[kStaticScratchBytes];

namespace {

dsv4kv_status scratch_address(void** out, const char* what) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_index_scratch);
  if (e != cudaSuccess || !p)
    return set_error(DSV4KV_ERR_CUDA, "%s: cudaGetSymbolAddress: %s", what, cudaGetErrorString(e));
  *out = p;
  return DSV4KV_OK;
}

}  // namespace
}  // namespace dsv4kv

using namespace dsv4kv;

extern "C" __attribute__((visibility("default"))) size_t dsv4kv_index_topk_noalloc_max_scratch_bytes(void) {
  return kStaticScratchBytes;
}

extern "C" __attribute__((visibility("default"))) dsv4kv_status dsv4kv_index_topk_noalloc(
    const void* qidx, const dsv4kv_cache* keys, int32_t batch, int64_t n, int32_t k, int32_t* idx_out,
    int32_t* count_out, void* stream) {
  if (batch < 0 || n < 0) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_noalloc: bad sizes");
  if (k < 1 || k > 2048) return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_noalloc: k must be in [1, 2048]");
  const size_t need = dsv4kv_index_topk_workspace_bytes(batch, n, k);
  if (need > kStaticScratchBytes)
    return set_error(DSV4KV_ERR_UNSUPPORTED,
                     "index_topk_noalloc: this call needs %zu bytes of scratch, above the %zu-byte static maximum "
                     "(use dsv4kv_index_topk with a workspace)",
                     need, kStaticScratchBytes);
  void* ws = nullptr;
  if (batch > 0 && n > k) {
    dsv4kv_status st = scratch_address(&ws, "index_topk_noalloc");
    if (st != DSV4KV_OK) return st;
    // After the status word the layout holds the per-sequence histograms and
    // the score kernel's claim counter; a successful call leaves them zero,
    // but one that gave up may not have, so clear them.
    const size_t zero_bytes = index_topk_zero_prefix_bytes(batch);
    if (zero_bytes <= kStatusBytes || zero_bytes > need)
      return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_noalloc: bad scratch layout (%zu bytes to clear)", zero_bytes);
    const cudaError_t e = cudaMemsetAsync(static_cast<char*>(ws) + kStatusBytes, 0, zero_bytes - kStatusBytes,
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
      return set_error(DSV4KV_ERR_CUDA, "index_topk_noalloc: clearing scratch: %s", cudaGetErrorString(e));
  }
  return dsv4kv_index_topk(qidx, keys, batch, n, k, idx_out, count_out, ws, kStaticScratchBytes, stream);
}

extern "C" __attribute__((visibility("default"))) dsv4kv_status dsv4kv_index_topk_noalloc_status(
    uint32_t* host_out, int32_t clear, void* stream) {
  if (!host_out) return set_error(DSV4KV_ERR_INVALID_ARG, "index_topk_noalloc_status: host_out is null");
  void* ws = nullptr;
  dsv4kv_status st = scratch_address(&ws, "index_topk_noalloc_status");
  if (st != DSV4KV_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess)
    return set_error(DSV4KV_ERR_CUDA, "index_topk_noalloc_status: %s", cudaGetErrorString(e));
  return DSV4KV_OK;
}
