// Incremental cache maintenance for one decode step (the steps either side
// of the path; [P1] "compressor-state blocks").
//
// After the state of position t is appended, one layer's caches hold
//   * raw ring  (bf16 [B][W+K][D]): row p % (W+K) = the unrotated state S[p]
//     for the last W + K positions (what the next entries still mix);
//   * window ring (bf16 [B][W][D]): row p % W = rope(S[p], p) for the last W
//     positions (the decode's window rows; their order does not matter to it);
//   * compressed cache (bf16 [B][rows][D]): entries 0 .. N(t+1) - 1, the new
//     one emitted the step its stride block [s i, s i + s) leaves the window,
//     N(t) = max(0, floor((t - W) / s)).
// An entry mixes positions s i + s - K + j (j < K, positions < 0 are zero)
// with the per-tap, per-channel weights w[j][c], then rotates its rotary
// pairs at position s i ([P1] "c4a (the milder scheme)", "c128a (the
// aggressive scheme)"; [P2] Step 4).  Its taps all lie in the last W + K
// positions, so the raw ring is enough.
//
// One CTA of 8 warps per sequence; lane l of a warp owns channels
// [PER l, PER l + PER).  Warp 0 writes the raw and window rows; when an entry
// is due, warp w sums the taps j = w, w + 8, ... and the warps' sums are
// added in warp order through shared memory before the rotation.  The
// rotation uses an fp64 angle reduced exactly modulo 2 pi (as the batch
// compressor); the cos / sin of every rotary pair at the window row's and at
// the entry's position are computed once per CTA, one pair per lane, by
// warps 1 and 2 while warp 0 copies the raw row (each is a dependent chain of
// double-precision work; the lanes that own the rotary channels would
// otherwise run 8 of them one after another).
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

namespace {

constexpr int kAppendWarps = 8;

// cos / sin of the angle pos * rope_base^(-2m / rope_dim) of every rotary
// pair m, the angle in units of pi reduced exactly modulo 2; lane l takes
// pairs l, l + 32, ...
__device__ __forceinline__ void rope_table(double* cs, double* sn, int rope_dim, double rope_base, double pos,
                                           int lane) {
  for (int m = lane; m < rope_dim / 2; m += 32) {
    const double ang = pos * (pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793);
    const double xr = ang - 2.0 * rint(0.5 * ang);
    sincospi(xr, &sn[m], &cs[m]);
  }
}

template <int PER>
__device__ __forceinline__ void rope_pairs(float (&v)[PER], int c0, int dim, int rope_dim, const double* cs,
                                           const double* sn) {
  const int r0 = dim - rope_dim;
  if (c0 + PER <= r0) return;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const int c = c0 + e;
    if (c >= r0) {
      const int m = (c - r0) >> 1;
      const float x = v[e], y = v[e + 1];
      v[e] = float(double(x) * cs[m] - double(y) * sn[m]);
      v[e + 1] = float(double(x) * sn[m] + double(y) * cs[m]);
    }
  }
}

template <int PER>
__device__ __forceinline__ void store_bf16_row(uint16_t* dst, const float (&v)[PER]) {
#pragma unroll
  for (int q = 0; q < PER / 8; ++q)
    *reinterpret_cast<uint4*>(dst + 8 * q) =
        make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                   pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

template <int PER>
__global__ void __launch_bounds__(32 * kAppendWarps)
    append_kernel(const uint16_t* __restrict__ s_new, const float* __restrict__ w, int64_t t, int k_taps, int stride,
                  int window, int rope_dim, double rope_base, uint16_t* __restrict__ raw_ring,
                  uint16_t* __restrict__ win_ring, uint16_t* __restrict__ comp, int64_t comp_rows, int64_t emit) {
  constexpr int D = 32 * PER;
  __shared__ __align__(16) float red[kAppendWarps][D];
  extern __shared__ double rtab[];  // cos, sin at the window row's position; cos, sin at the entry's
  const int np = rope_dim / 2;
  double* w_cs = rtab;
  double* w_sn = rtab + np;
  double* e_cs = rtab + 2 * np;
  double* e_sn = rtab + 3 * np;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int c0 = PER * lane;
  const int64_t ring = int64_t(window) + k_taps;
  const uint16_t* xs = s_new + size_t(b) * D + c0;
  pdl_trigger();
  pdl_wait();
  uint4 raw[PER / 8];
  if (warp == 0) {
#pragma unroll
    for (int q = 0; q < PER / 8; ++q) raw[q] = *reinterpret_cast<const uint4*>(xs + 8 * q);
    uint16_t* rr = raw_ring + (size_t(b) * size_t(ring) + size_t(t % ring)) * D + c0;
#pragma unroll
    for (int q = 0; q < PER / 8; ++q) *reinterpret_cast<uint4*>(rr + 8 * q) = raw[q];
  }
  if (warp == 1 && window > 0) rope_table(w_cs, w_sn, rope_dim, rope_base, double(t), lane);
  if (warp == 2 && emit >= 0) rope_table(e_cs, e_sn, rope_dim, rope_base, double(int64_t(stride) * emit), lane);
  __syncthreads();
  if (warp == 0) {
    if (window > 0) {
      float v[PER];
#pragma unroll
      for (int q = 0; q < PER / 8; ++q) {
        v[8 * q] = bf16lo(raw[q].x); v[8 * q + 1] = bf16hi(raw[q].x);
        v[8 * q + 2] = bf16lo(raw[q].y); v[8 * q + 3] = bf16hi(raw[q].y);
        v[8 * q + 4] = bf16lo(raw[q].z); v[8 * q + 5] = bf16hi(raw[q].z);
        v[8 * q + 6] = bf16lo(raw[q].w); v[8 * q + 7] = bf16hi(raw[q].w);
      }
      rope_pairs<PER>(v, c0, D, rope_dim, w_cs, w_sn);
      store_bf16_row<PER>(win_ring + (size_t(b) * size_t(window) + size_t(t % window)) * D + c0, v);
    }
  }
  if (emit < 0) return;  // block-uniform
  // this warp's taps of entry `emit`
  const int64_t first = int64_t(stride) * emit + stride - k_taps;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll 2
  for (int j = warp; j < k_taps; j += kAppendWarps) {
    const int64_t pos = first + j;
    if (pos < 0) continue;
    // the newest position is read from the input (warp 0 may still be writing its ring row)
    const uint16_t* row = pos == t ? xs : raw_ring + (size_t(b) * size_t(ring) + size_t(pos % ring)) * D + c0;
    const float* wr = w + size_t(j) * D + c0;
#pragma unroll
    for (int q = 0; q < PER / 8; ++q) {
      const uint4 x = *reinterpret_cast<const uint4*>(row + 8 * q);
      const float4 wa = *reinterpret_cast<const float4*>(wr + 8 * q);
      const float4 wb = *reinterpret_cast<const float4*>(wr + 8 * q + 4);
      acc[8 * q + 0] = fmaf(wa.x, bf16lo(x.x), acc[8 * q + 0]);
      acc[8 * q + 1] = fmaf(wa.y, bf16hi(x.x), acc[8 * q + 1]);
      acc[8 * q + 2] = fmaf(wa.z, bf16lo(x.y), acc[8 * q + 2]);
      acc[8 * q + 3] = fmaf(wa.w, bf16hi(x.y), acc[8 * q + 3]);
      acc[8 * q + 4] = fmaf(wb.x, bf16lo(x.z), acc[8 * q + 4]);
      acc[8 * q + 5] = fmaf(wb.y, bf16hi(x.z), acc[8 * q + 5]);
      acc[8 * q + 6] = fmaf(wb.z, bf16lo(x.w), acc[8 * q + 6]);
      acc[8 * q + 7] = fmaf(wb.w, bf16hi(x.w), acc[8 * q + 7]);
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) red[warp][c0 + e] = acc[e];
  __syncthreads();
  if (warp != 0) return;
  float v[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    float sum = red[0][c0 + e];
#pragma unroll
    for (int ww = 1; ww < kAppendWarps; ++ww) sum += red[ww][c0 + e];
    v[e] = sum;
  }
  rope_pairs<PER>(v, c0, D, rope_dim, e_cs, e_sn);
  store_bf16_row<PER>(comp + (size_t(b) * size_t(comp_rows) + size_t(emit)) * D + c0, v);
}

}  // namespace

int64_t append_emit_entry(int64_t t, int window, int stride) {
  const int64_t n0 = t >= window ? (t - window) / stride : 0;
  const int64_t n1 = t + 1 >= window ? (t + 1 - window) / stride : 0;
  return n1 > n0 ? n1 - 1 : -1;
}

dsv4kv_status append_launch(const void* s_new, const float* w, int batch, int64_t t, int dim, int k_taps, int stride,
                            int window, int rope_dim, double rope_base, void* raw_ring, void* win_ring, void* comp,
                            int64_t comp_rows, cudaStream_t stream) {
  const int64_t emit = append_emit_entry(t, window, stride);
  const uint16_t* s = static_cast<const uint16_t*>(s_new);
  uint16_t* rr = static_cast<uint16_t*>(raw_ring);
  uint16_t* wr = static_cast<uint16_t*>(win_ring);
  uint16_t* cp = static_cast<uint16_t*>(comp);
  const dim3 grid{static_cast<unsigned>(batch)}, block{32 * kAppendWarps};
  const size_t tab = size_t(rope_dim / 2) * 4 * sizeof(double);  // two positions x (cos, sin) per rotary pair
  switch (dim) {
    case 256:
      launch_pdl(append_kernel<8>, grid, block, tab, stream, s, w, t, k_taps, stride, window, rope_dim, rope_base, rr,
                 wr, cp, comp_rows, emit);
      break;
    case 512:
      launch_pdl(append_kernel<16>, grid, block, tab, stream, s, w, t, k_taps, stride, window, rope_dim, rope_base, rr,
                 wr, cp, comp_rows, emit);
      break;
    case 1024:
      launch_pdl(append_kernel<32>, grid, block, tab, stream, s, w, t, k_taps, stride, window, rope_dim, rope_base, rr,
                 wr, cp, comp_rows, emit);
      break;
    default:
      return set_error(DSV4KV_ERR_UNSUPPORTED, "append: dim must be 256, 512 or 1024 (got %d)", dim);
  }
  return check_launch("append_kernel");
}

}  // namespace dsv4kv
