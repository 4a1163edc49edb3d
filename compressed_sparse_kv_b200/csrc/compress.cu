// c4a / c128a compressors.
//
// [P1] "c4a (the milder scheme)": each compressed entry is a learned weighted
// sum of 8 states, the next entry shifted by 4; "c128a (the aggressive
// scheme)": 128 states at stride 128.  [P2] Step 4: C4A[1] = mix(S0..S7),
// C4A[2] = mix(S4..S11), C128A[0] = mix(S0..S127).  Entry i of stride s with
// K taps mixes positions s*i + s - K + j (j < K; positions < 0 contribute 0),
// per channel, then rotates its rotary channel pairs at position pos0 + s*i.
//
// Layout of the work (compress_kernel; at dim 512, c4a uses compress_c4_kernel
// and c128a compress_c128_kernel, below): one warp per entry, each lane owns 16 consecutive channels (two
// 16-byte bf16 loads per tap row), so a tap row is one fully coalesced 1 KB
// read.  The K tap loads are unrolled by 4 to keep several
// rows in flight; c4a entries overlap by 4 rows, which the L1/L2 absorb.
// The rotation: the block computes rope_base^(-2m/rope_dim) / pi once per
// pair m (shared memory); per entry, lane m computes the cos / sin of pair m
// (the angle in units of pi reduced exactly modulo 2 in fp64, then sincospi)
// and the lanes that own rotary channels take theirs by shuffles.
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kMaxRopePairs = 512;  // rope_dim <= 1024

template <int PER>  // channels per lane (dim / 32)
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
    compress_kernel(const uint16_t* __restrict__ s_raw, const float* __restrict__ w, int64_t t, int k_taps,
                    int stride, int64_t n_entries, int64_t pos0, int rope_dim, double rope_base, int out_fp32,
                    void* __restrict__ out) {
  constexpr int D = 32 * PER;
  __shared__ double theta_pi[kMaxRopePairs];  // rope_base^(-2m/rope_dim) / pi
  for (int m = threadIdx.x; m < rope_dim / 2; m += blockDim.x)
    theta_pi[m] = pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int64_t i = int64_t(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (i >= n_entries) return;
  const int c0 = PER * lane;
  const uint16_t* sb = s_raw + size_t(b) * size_t(t) * D + c0;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const int64_t first = int64_t(stride) * i + stride - k_taps;
  const int j0 = first < 0 ? int(-first) : 0;  // skip taps before position 0
#pragma unroll 4
  for (int j = j0; j < k_taps; ++j) {
    const uint16_t* row = sb + size_t(first + j) * D;
    const float* wr = w + size_t(j) * D + c0;
#pragma unroll
    for (int v = 0; v < PER / 8; ++v) {
      const uint4 x = *reinterpret_cast<const uint4*>(row + 8 * v);
      const float4 wa = *reinterpret_cast<const float4*>(wr + 8 * v);
      const float4 wb = *reinterpret_cast<const float4*>(wr + 8 * v + 4);
      acc[8 * v + 0] = fmaf(wa.x, bf16lo(x.x), acc[8 * v + 0]);
      acc[8 * v + 1] = fmaf(wa.y, bf16hi(x.x), acc[8 * v + 1]);
      acc[8 * v + 2] = fmaf(wa.z, bf16lo(x.y), acc[8 * v + 2]);
      acc[8 * v + 3] = fmaf(wa.w, bf16hi(x.y), acc[8 * v + 3]);
      acc[8 * v + 4] = fmaf(wb.x, bf16lo(x.z), acc[8 * v + 4]);
      acc[8 * v + 5] = fmaf(wb.y, bf16hi(x.z), acc[8 * v + 5]);
      acc[8 * v + 6] = fmaf(wb.z, bf16lo(x.w), acc[8 * v + 6]);
      acc[8 * v + 7] = fmaf(wb.w, bf16hi(x.w), acc[8 * v + 7]);
    }
  }
  // RoPE at the block's first position.  The pair index m of channel c is
  // (c - (D - rope_dim)) / 2; the angle pos * theta_m in units of pi is
  // reduced exactly modulo 2 (fp64) before sincospi.
  const int r0 = D - rope_dim;
  const int pairs = rope_dim / 2;
  const double pos = double(pos0 + int64_t(stride) * i);
  auto rotation = [&](int m, float* cs, float* sn) {
    const double ang = pos * theta_pi[m];
    double sd, cd;
    sincospi(ang - 2.0 * rint(0.5 * ang), &sd, &cd);
    *cs = float(cd);
    *sn = float(sd);
  };
  if (pairs <= 32) {
    // lane m computes pair m; the owners of rotary channels fetch theirs
    float cs_m = 1.f, sn_m = 0.f;
    if (lane < pairs) rotation(lane, &cs_m, &sn_m);
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const int c = c0 + e;
      const int m = c >= r0 ? (c - r0) >> 1 : 0;
      const float cs = __shfl_sync(kFull, cs_m, m & 31), sn = __shfl_sync(kFull, sn_m, m & 31);
      if (c >= r0) {
        const float x = acc[e], y = acc[e + 1];
        acc[e] = float(double(x) * cs - double(y) * sn);
        acc[e + 1] = float(double(x) * sn + double(y) * cs);
      }
    }
  } else if (c0 + PER > r0) {
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const int c = c0 + e;
      if (c >= r0) {
        float cs, sn;
        rotation((c - r0) >> 1, &cs, &sn);
        const float x = acc[e], y = acc[e + 1];
        acc[e] = float(double(x) * cs - double(y) * sn);
        acc[e + 1] = float(double(x) * sn + double(y) * cs);
      }
    }
  }
  const size_t o = (size_t(b) * size_t(n_entries) + size_t(i)) * D + c0;
  if (out_fp32) {
    float* op = static_cast<float*>(out) + o;
#pragma unroll
    for (int v = 0; v < PER / 4; ++v)
      *reinterpret_cast<float4*>(op + 4 * v) = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
  } else {
    uint16_t* op = static_cast<uint16_t*>(out) + o;
#pragma unroll
    for (int v = 0; v < PER / 8; ++v)
      *reinterpret_cast<uint4*>(op + 8 * v) =
          make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                     pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
  }
}


// c4a-shaped compression (K taps at stride S = K / 2, dim 512), with each
// warp emitting consecutive entries: entry i mixes rows [S(i-1), S(i+1)), so
// row r feeds entry floor(r / S) (taps S..K-1) and the next one (taps
// 0..S-1).  A CTA of four warps takes kC4Entries consecutive entries of one
// sequence; warp w owns channels [128 w, 128 w + 128), 4 per lane, whose K x 4
// weights stay in registers.  The warp walks its rows once, block by block of
// S rows (the next block's loads issued before the current one is used),
// keeping two accumulators: the entry being completed and the next one.  The
// taps of an entry are added in ascending order, as in compress_kernel, so
// the results are the same bit for bit.
constexpr int kC4Entries = 32;

template <int K>
__global__ void __launch_bounds__(128) compress_c4_kernel(const uint16_t* __restrict__ s_raw,
                                                          const float* __restrict__ w, int64_t t, int64_t n_entries,
                                                          int64_t pos0, int rope_dim, double rope_base, int out_fp32,
                                                          void* __restrict__ out) {
  constexpr int S = K / 2, D = 512;
  __shared__ double theta_pi[kMaxRopePairs];  // rope_base^(-2m/rope_dim) / pi
  for (int m = threadIdx.x; m < rope_dim / 2; m += blockDim.x)
    theta_pi[m] = pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int64_t i0 = int64_t(blockIdx.x) * kC4Entries;
  const int64_t i1 = min(n_entries, i0 + kC4Entries);
  if (i0 >= i1) return;
  const int c = 128 * warp + 4 * lane;  // this lane's 4 channels
  float wr[K][4];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const float4 x = *reinterpret_cast<const float4*>(w + size_t(j) * D + c);
    wr[j][0] = x.x;
    wr[j][1] = x.y;
    wr[j][2] = x.z;
    wr[j][3] = x.w;
  }
  const uint16_t* sb = s_raw + size_t(b) * size_t(t) * D + c;
  auto load_block = [&](int64_t q, uint2 (&v)[S]) {
#pragma unroll
    for (int u = 0; u < S; ++u) {
      const int64_t r = S * q + u;
      v[u] = r >= 0 ? *reinterpret_cast<const uint2*>(sb + size_t(r) * D) : make_uint2(0, 0);
    }
  };
  const int r0 = D - rope_dim;
  float acc_a[4] = {0.f, 0.f, 0.f, 0.f}, acc_b[4] = {0.f, 0.f, 0.f, 0.f};
  uint2 cur[S], nxt[S] = {};
  int64_t q = i0 - 1;  // block q = rows [S q, S q + S): taps S.. of entry q, taps 0.. of entry q + 1
  load_block(q, cur);
  for (; q < i1; ++q) {
    if (q + 1 < i1) load_block(q + 1, nxt);
#pragma unroll
    for (int u = 0; u < S; ++u) {
      if (S * q + u < 0) continue;  // positions before 0 contribute nothing
      const float x[4] = {bf16lo(cur[u].x), bf16hi(cur[u].x), bf16lo(cur[u].y), bf16hi(cur[u].y)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc_a[e] = fmaf(wr[S + u][e], x[e], acc_a[e]);
        acc_b[e] = fmaf(wr[u][e], x[e], acc_b[e]);
      }
    }
    if (q >= i0) {  // entry q is complete: rotate its rotary pairs at position pos0 + S q, store
      if (c + 4 > r0) {
        const double pos = double(pos0 + int64_t(S) * q);
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          if (c + e >= r0) {
            const double ang = pos * theta_pi[(c + e - r0) >> 1];
            double sd, cd;
            sincospi(ang - 2.0 * rint(0.5 * ang), &sd, &cd);
            const float cs = float(cd), sn = float(sd);
            const float xa = acc_a[e], ya = acc_a[e + 1];
            acc_a[e] = float(double(xa) * cs - double(ya) * sn);
            acc_a[e + 1] = float(double(xa) * sn + double(ya) * cs);
          }
        }
      }
      const size_t o = (size_t(b) * size_t(n_entries) + size_t(q)) * D + c;
      if (out_fp32)
        *reinterpret_cast<float4*>(static_cast<float*>(out) + o) = make_float4(acc_a[0], acc_a[1], acc_a[2], acc_a[3]);
      else
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + o) =
            make_uint2(pack_bf16x2(acc_a[0], acc_a[1]), pack_bf16x2(acc_a[2], acc_a[3]));
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc_a[e] = acc_b[e];
      acc_b[e] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < S; ++u) cur[u] = nxt[u];
  }
}


// c128a-shaped compression (K taps at stride S = K, K a multiple of 16, dim
// 512): entries do not share rows, and the K x 512 fp32 weights (256 KB for
// K = 128) are what every entry re-reads.  A CTA of kC128Groups groups of
// four warps takes kC128Entries consecutive entries of one sequence, each
// group a quarter of them; warp w of a group owns channels [128 w, 128 w +
// 128), 4 per lane, and keeps the accumulators of its entries in registers.
// The weights come through shared memory 16 taps (32 KB) at a time, so each
// weight is read from L2 once per CTA instead of once per entry; the rows
// stream with 16 loads in flight per lane.  (Bulk c128a, B=8 t=131072, 16
// entries and 16-tap chunks: 182 us with four groups, 226 with two, 230 with
// eight, 288 with one; 211 us with four groups of 8 entries; one warp per
// entry with the weights from L2 387 us.)
// Taps are added in ascending order, as in compress_kernel, so the results
// are the same bit for bit.
constexpr int kC128Entries = 16;
constexpr int kC128Groups = 4;  // groups of four warps, each taking kC128Entries / kC128Groups of the entries
constexpr int kC128Chunk = 16;  // taps per staged weight chunk (the rows go in batches of 16 taps)
static_assert(kC128Chunk % 16 == 0, "whole batches of 16 taps per chunk");

__global__ void __launch_bounds__(128 * kC128Groups) compress_c128_kernel(const uint16_t* __restrict__ s_raw,
                                                            const float* __restrict__ w, int64_t t, int k_taps,
                                                            int64_t n_entries, int64_t pos0, int rope_dim,
                                                            double rope_base, int out_fp32, void* __restrict__ out) {
  constexpr int D = 512, E = kC128Entries / kC128Groups, J = kC128Chunk;
  extern __shared__ __align__(16) float w_s[];  // [J][D]
  __shared__ double theta_pi[kMaxRopePairs];
  for (int m = threadIdx.x; m < rope_dim / 2; m += blockDim.x)
    theta_pi[m] = pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int64_t i0 = int64_t(blockIdx.x) * kC128Entries + int64_t(warp >> 2) * E;  // this warp's entries
  const int ne = int(max(int64_t(0), min(int64_t(E), n_entries - i0)));
  const int c = 128 * (warp & 3) + 4 * lane;
  const int S = k_taps;
  const uint16_t* sb = s_raw + size_t(b) * size_t(t) * D + c;
  float acc[E][4];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e][0] = acc[e][1] = acc[e][2] = acc[e][3] = 0.f;
  for (int jc = 0; jc < k_taps; jc += J) {
    __syncthreads();  // the previous chunk's weights have been used
    for (int v = threadIdx.x; v < J * D / 4; v += blockDim.x)
      reinterpret_cast<float4*>(w_s)[v] = reinterpret_cast<const float4*>(w + size_t(jc) * D)[v];
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (e >= ne) continue;
      const uint16_t* rows = sb + (size_t(S) * size_t(i0 + e) + size_t(jc)) * D;  // tap jc of entry i0 + e
#pragma unroll
      for (int h = 0; h < J; h += 16) {
        uint2 x[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) x[u] = *reinterpret_cast<const uint2*>(rows + size_t(h + u) * D);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 wv = *reinterpret_cast<const float4*>(w_s + (h + u) * D + c);
          acc[e][0] = fmaf(wv.x, bf16lo(x[u].x), acc[e][0]);
          acc[e][1] = fmaf(wv.y, bf16hi(x[u].x), acc[e][1]);
          acc[e][2] = fmaf(wv.z, bf16lo(x[u].y), acc[e][2]);
          acc[e][3] = fmaf(wv.w, bf16hi(x[u].y), acc[e][3]);
        }
      }
    }
  }
  const int r0 = D - rope_dim;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (e >= ne) continue;
    const int64_t i = i0 + e;
    if (c + 4 > r0) {  // rotate the rotary pairs at position pos0 + S i
      const double pos = double(pos0 + int64_t(S) * i);
#pragma unroll
      for (int q = 0; q < 4; q += 2) {
        if (c + q >= r0) {
          const double ang = pos * theta_pi[(c + q - r0) >> 1];
          double sd, cd;
          sincospi(ang - 2.0 * rint(0.5 * ang), &sd, &cd);
          const float cs = float(cd), sn = float(sd);
          const float xa = acc[e][q], ya = acc[e][q + 1];
          acc[e][q] = float(double(xa) * cs - double(ya) * sn);
          acc[e][q + 1] = float(double(xa) * sn + double(ya) * cs);
        }
      }
    }
    const size_t o = (size_t(b) * size_t(n_entries) + size_t(i)) * D + c;
    if (out_fp32)
      *reinterpret_cast<float4*>(static_cast<float*>(out) + o) = make_float4(acc[e][0], acc[e][1], acc[e][2], acc[e][3]);
    else
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + o) =
          make_uint2(pack_bf16x2(acc[e][0], acc[e][1]), pack_bf16x2(acc[e][2], acc[e][3]));
  }
}

}  // namespace

dsv4kv_status compress_launch(const void* s_raw, const float* w, int batch, int64_t t, int dim, int k_taps,
                              int stride, int window, int64_t pos0, int rope_dim, double rope_base,
                              int out_fp32, void* out, cudaStream_t stream) {
  const int64_t n = std::max<int64_t>(0, (t - window) / stride);
  if (n == 0) return DSV4KV_OK;
  const uint16_t* s = static_cast<const uint16_t*>(s_raw);
  if (dim == 512 && k_taps == 8 && stride == 4) {  // c4a: consecutive entries per warp
    dim3 grid(unsigned((n + kC4Entries - 1) / kC4Entries), unsigned(batch));
    compress_c4_kernel<8><<<grid, 128, 0, stream>>>(s, w, t, n, pos0, rope_dim, rope_base, out_fp32, out);
    return check_launch("compress_c4_kernel");
  }
  if (dim == 512 && k_taps == stride && k_taps % kC128Chunk == 0) {  // c128a: weights staged per CTA
    static std::atomic<uint64_t> attr_set{0};
    constexpr int kSmem = kC128Chunk * 512 * int(sizeof(float));
    if (!done_on_device(attr_set)) {
      if (cudaFuncSetAttribute(compress_c128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
          cudaSuccess)
        return check_launch("compress: cudaFuncSetAttribute");
      mark_done_on_device(attr_set);
    }
    dim3 grid(unsigned((n + kC128Entries - 1) / kC128Entries), unsigned(batch));
    compress_c128_kernel<<<grid, 128 * kC128Groups, kSmem, stream>>>(s, w, t, k_taps, n, pos0, rope_dim, rope_base,
                                                                    out_fp32, out);
    return check_launch("compress_c128_kernel");
  }
  dim3 grid(unsigned((n + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned(batch));
  switch (dim) {
    case 256:
      compress_kernel<8><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(s, w, t, k_taps, stride, n, pos0, rope_dim,
                                                                  rope_base, out_fp32, out);
      break;
    case 512:
      compress_kernel<16><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(s, w, t, k_taps, stride, n, pos0, rope_dim,
                                                                   rope_base, out_fp32, out);
      break;
    case 1024:
      compress_kernel<32><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(s, w, t, k_taps, stride, n, pos0, rope_dim,
                                                                   rope_base, out_fp32, out);
      break;
    default:
      return set_error(DSV4KV_ERR_UNSUPPORTED, "compress: dim must be 256, 512 or 1024 (got %d)", dim);
  }
  return check_launch("compress_kernel");
}

}  // namespace dsv4kv
