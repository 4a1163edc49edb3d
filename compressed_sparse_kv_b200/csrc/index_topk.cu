// Lightning indexer scores and exact top-k selection.
//
// [P1] "c4a (the milder scheme)": DeepSeek Sparse Attention keeps the top-k
// (k = 512) compressed entries per query; [P1] indexer paragraph: the indexer
// cache holds 128 values per entry and may be fp4; [P2] Step 5: the learned
// indexer scores compressed blocks and the query reads the selected ones.
//
// Three launches per call (all on the caller's stream):
//  1. index_score_*: streams the keys once (16-byte vector loads, half a warp
//     per bf16 key / a quarter warp per fp4 key), writes one fp32 score per
//     entry to the workspace and builds a per-sequence histogram of the top
//     12 bits of the order-preserving score code.
//  2. index_filter_select: every CTA finds the threshold bin b1 of its
//     sequence from that histogram, appends every entry whose bin is >= b1 to
//     a candidate list, and builds a second-level histogram (next 12 bits) of
//     the entries in bin b1.  The last CTA of a sequence to finish (atomic
//     ticket, no waiting) resolves the exact selection from the candidates:
//     entries above the 24-bit threshold prefix are in; among the entries at
//     the prefix it orders by (score desc, index asc) and takes what is
//     missing; it sorts the selection by index, writes it, and re-zeroes the
//     sequence's histograms and counters.
//  3. (only when n <= k) index_fill_all writes 0..n-1 directly.
// The order (score desc, index asc) is a total order, so the result is the
// same for every split of the entries (exact, not approximate).
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

constexpr int kHistBins = 4096;  // 12-bit digits

// ------------------------------------------------------------------ scoring
// Transposing butterfly: lane l16 of a 16-lane group holds U partial sums
// (one per key); after log2 steps each lane holds the full 16-lane sum of one
// key.  U = 16: key l16 (15 shuffles for 16 keys).  U = 8: key (l16 >> 1) & 7,
// duplicated on lanes 2i and 2i+1 (8 shuffles for 8 keys).
template <int U>
__device__ __forceinline__ float reduce16_transposed(const float (&p)[U], int l16) {
  float a[8], c[4], d[2];
  if constexpr (U == 16) {
    const bool b3 = l16 & 8;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      a[i] = (b3 ? p[8 + i] : p[i]) + __shfl_xor_sync(kFull, b3 ? p[i] : p[8 + i], 8);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = p[i];
  }
  const int sh = U == 16 ? 0 : 1;  // lane bit that selects in the next step
  const bool x2 = (l16 >> (2 + sh)) & 1, x1 = (l16 >> (1 + sh)) & 1, x0 = (l16 >> sh) & 1;
  const int o2 = 4 << sh, o1 = 2 << sh, o0 = 1 << sh;
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = (x2 ? a[4 + i] : a[i]) + __shfl_xor_sync(kFull, x2 ? a[i] : a[4 + i], o2);
#pragma unroll
  for (int i = 0; i < 2; ++i) d[i] = (x1 ? c[2 + i] : c[i]) + __shfl_xor_sync(kFull, x1 ? c[i] : c[2 + i], o1);
  float s = (x0 ? d[1] : d[0]) + __shfl_xor_sync(kFull, x0 ? d[0] : d[1], o0);
  if constexpr (U == 8) s += __shfl_xor_sync(kFull, s, 1);
  return s;
}

__device__ __forceinline__ float dot8_bf16(const uint4& v, const float (&q)[8]) {
  float a = q[0] * bf16lo(v.x);
  a = fmaf(q[1], bf16hi(v.x), a);
  a = fmaf(q[2], bf16lo(v.y), a);
  a = fmaf(q[3], bf16hi(v.y), a);
  a = fmaf(q[4], bf16lo(v.z), a);
  a = fmaf(q[5], bf16hi(v.z), a);
  a = fmaf(q[6], bf16lo(v.w), a);
  return fmaf(q[7], bf16hi(v.w), a);
}

// bf16 keys, dim 128: a key is 256 B = 16 lanes x 16 B.  The flattened
// (sequence, entry) range of all B*n keys is split evenly over the grid; a
// CTA walks its range one sequence segment at a time.  A warp iteration
// covers 2U keys: half-warp h reads keys 2U*j + U*h + u (u < U), U
// independent 16-byte loads per lane; with DB the next iteration's loads are
// issued before the current iteration is reduced, so loads stay in flight.
template <int U, bool DB>
__global__ void __launch_bounds__(256) index_score_bf16(const uint16_t* __restrict__ qidx,
                                                        const uint16_t* __restrict__ keys, int64_t key_rows,
                                                        int64_t n, int batch, int64_t per_cta,
                                                        float* __restrict__ scores, uint32_t* __restrict__ hist) {
  __shared__ uint32_t sh[kHistBins];
  pdl_trigger();
  const int64_t total = int64_t(batch) * n;
  const int64_t g0 = int64_t(blockIdx.x) * per_cta;
  const int64_t g1 = min(total, g0 + per_cta);
  if (g0 >= g1) return;
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int half = lane >> 4, l16 = lane & 15;
  const int my_key = U == 16 ? l16 : ((l16 >> 1) & 7);
  const bool writer = U == 16 || !(lane & 1);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0;
  for (int64_t s0 = g0; s0 < g1;) {
    const int b = int(s0 / n);
    const int64_t s1 = min(g1, int64_t(b + 1) * n);
    const int64_t i0 = s0 - int64_t(b) * n, cnt = s1 - s0;
    float q[8];
    {
      const uint4 v = *reinterpret_cast<const uint4*>(qidx + size_t(b) * 128 + 8 * l16);
      q[0] = bf16lo(v.x); q[1] = bf16hi(v.x); q[2] = bf16lo(v.y); q[3] = bf16hi(v.y);
      q[4] = bf16lo(v.z); q[5] = bf16hi(v.z); q[6] = bf16lo(v.w); q[7] = bf16hi(v.w);
    }
    __syncthreads();  // histogram cleared
    const uint16_t* kb = keys + (size_t(b) * size_t(key_rows) + size_t(i0)) * 128 + 8 * l16;
    float* sc = scores + size_t(b) * size_t(n) + size_t(i0);
    auto load = [&](int64_t j, uint4 (&v)[U]) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t key = 2 * U * j + U * half + u;
        v[u] = key < cnt ? ld_stream_v4(kb + key * 128) : make_uint4(0, 0, 0, 0);
      }
    };
    auto process = [&](int64_t j, const uint4 (&v)[U]) {
      float p[U];
#pragma unroll
      for (int u = 0; u < U; ++u) p[u] = dot8_bf16(v[u], q);
      const float s = reduce16_transposed<U>(p, l16) + 0.0f;  // -0 -> +0
      const int64_t key = 2 * U * j + U * half + my_key;
      if (writer && key < cnt) {
        sc[key] = s;
        atomicAdd(&sh[ord_f32(s) >> 20], 1u);
      }
    };
    const int64_t ngroups = (cnt + 2 * U - 1) / (2 * U);
    if constexpr (DB) {
      uint4 va[U], vb[U];
      int64_t j = warp;
      if (j < ngroups) load(j, va);
      while (j < ngroups) {
        if (j + nwarps < ngroups) load(j + nwarps, vb);
        process(j, va);
        j += nwarps;
        if (j >= ngroups) break;
        if (j + nwarps < ngroups) load(j + nwarps, va);
        process(j, vb);
        j += nwarps;
      }
    } else {
      for (int64_t j = warp; j < ngroups; j += nwarps) {
        uint4 v[U];
        load(j, v);
        process(j, v);
      }
    }
    __syncthreads();
    uint32_t* hb = hist + size_t(b) * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
      const uint32_t c = sh[i];
      if (c) {
        atomicAdd(&hb[i], c);
        sh[i] = 0;
      }
    }
    s0 = s1;
  }
}

// fp4 keys, dim 128: codes 64 B + 8 E4M3 scale bytes per key.  A quarter warp
// (4 lanes x 16 B) covers one key; each lane holds 32 channels = 2 scale
// groups.  E2M1 codes are decoded to packed f16 pairs with byte permutes
// (a PRMT table of the eight magnitudes) and the sign bit OR-ed in; each
// 16-channel group is accumulated with packed f16 FMAs (exact for integer
// queries: |partial| <= 16*8*6 = 768 at a resolution of 0.5 needs 11 bits)
// and the group sum is scaled in fp32.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// High bytes of the f16 encodings of 0, .5, 1, 1.5, 2, 3, 4, 6.
constexpr uint32_t kE2M1HiLo = 0x3E3C3800u;  // codes 3..0
constexpr uint32_t kE2M1HiHi = 0x46444240u;  // codes 7..4

// Decode the 8 nibbles of w into four f16x2: out[i] = (nibble i, nibble i+4).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&out)[4]) {
  const uint32_t mlo = prmt(kE2M1HiLo, kE2M1HiHi, w & 0x7777u);          // mags of nibbles 0..3
  const uint32_t mhi = prmt(kE2M1HiLo, kE2M1HiHi, (w >> 16) & 0x7777u);  // mags of nibbles 4..7
  // selector nibble 8 (sign-replicate of a byte whose top bit is 0) yields 0x00
  out[0] = prmt(mlo, mhi, 0x4808u) | ((w << 12) & 0x80008000u);
  out[1] = prmt(mlo, mhi, 0x5818u) | ((w << 8) & 0x80008000u);
  out[2] = prmt(mlo, mhi, 0x6828u) | ((w << 4) & 0x80008000u);
  out[3] = prmt(mlo, mhi, 0x7838u) | (w & 0x80008000u);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  // exact: E4M3 bits placed in a binary32 with the exponent rebased by 2^120
  const uint32_t mag = (c & 0x7fu) << 20;
  const float v = __uint_as_float(mag) * 0x1p120f;
  return (c & 0x80u) ? -v : v;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ float f16x2_sum(uint32_t h) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return lo + hi;
}
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}

__global__ void __launch_bounds__(256) index_score_fp4(const uint16_t* __restrict__ qidx,
                                                       const uint8_t* __restrict__ codes,
                                                       const uint8_t* __restrict__ scales, int64_t key_rows,
                                                       int64_t n, int64_t chunk, float* __restrict__ scores,
                                                       uint32_t* __restrict__ hist) {
  __shared__ uint32_t sh[kHistBins];
  pdl_trigger();
  const int b = blockIdx.y;
  const int64_t n0 = int64_t(blockIdx.x) * chunk;
  const int64_t n1 = min(n, n0 + chunk);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0;
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int quad = lane >> 2, l4 = lane & 3;  // key slot in the warp, segment in the key
  // Lane l4 covers channels [32*l4, 32*l4+32).  Word j of its 16 B holds
  // channels 32*l4 + 8j .. +8 (nibble e = channel 8j+e); the decode pairs
  // nibbles (i, i+4), so q is packed the same way: qp[j][i] = (q[8j+i], q[8j+i+4]).
  uint32_t qp[4][4];
  {
    const uint16_t* qb = qidx + size_t(b) * 128 + 32 * l4;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) qp[j][i] = f32x2_to_f16x2(bf16f(qb[8 * j + i]), bf16f(qb[8 * j + i + 4]));
  }
  __syncthreads();
  const uint8_t* cb = codes + size_t(b) * size_t(key_rows) * 64 + 16 * l4;
  const uint8_t* sb = scales + size_t(b) * size_t(key_rows) * 8 + 2 * l4;
  float* sc = scores + size_t(b) * size_t(n);
  constexpr int U = 4;  // keys per quad per iteration (32 keys per warp)
  for (int64_t base = n0 + 32 * warp; base < n1; base += 32 * nwarps) {
    uint4 v[U];
    uint32_t s2[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t key = base + 8 * u + quad;
      const bool ok = key < n1;
      v[u] = ok ? ld_stream_v4(cb + key * 64) : make_uint4(0, 0, 0, 0);
      s2[u] = ok ? *reinterpret_cast<const uint16_t*>(sb + key * 8) : 0u;
    }
    float p[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t acc0 = 0, acc1 = 0;  // f16x2 accumulators of group 0 (words 0,1) and group 1 (words 2,3)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t h[4];
        e2m1x8_to_f16x2(w[j], h);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (j < 2) acc0 = hfma2(qp[j][i], h[i], acc0);
          else acc1 = hfma2(qp[j][i], h[i], acc1);
        }
      }
      p[u] = f16x2_sum(acc0) * e4m3_to_f32(s2[u] & 0xffu) + f16x2_sum(acc1) * e4m3_to_f32(s2[u] >> 8);
    }
    // reduce over the 4 lanes of the quad: 4 values -> transposing butterfly
    const bool bb1 = l4 & 2, bb0 = l4 & 1;
    float k2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float keep = bb1 ? p[2 + i] : p[i];
      const float send = bb1 ? p[i] : p[2 + i];
      k2[i] = keep + __shfl_xor_sync(kFull, send, 2);
    }
    const float s = (bb0 ? k2[1] : k2[0]) + __shfl_xor_sync(kFull, bb0 ? k2[0] : k2[1], 1);
    const int64_t key = base + 8 * (2 * (l4 >> 1) + (l4 & 1)) + quad;
    if (key < n1) {
      const float sz = s + 0.0f;
      sc[key] = sz;
      atomicAdd(&sh[ord_f32(sz) >> 20], 1u);
    }
  }
  __syncthreads();
  uint32_t* hb = hist + size_t(b) * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&hb[i], sh[i]);
}

// ------------------------------------------------------------------ selection helpers
constexpr int kSelThreads = 512;
constexpr int kTieCap = 2048;
constexpr int64_t kMaxBitmapN = 262144;  // entries covered by the shared-memory bitmaps (8192 words each)

// Block-wide exclusive prefix sum of one value per thread (kSelThreads threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* total) {
  __shared__ uint32_t wsum[kSelThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const uint32_t x = wsum[w];
    base += w < warp ? x : 0u;
    all += x;
  }
  __syncthreads();
  if (total) *total = all;
  return base + incl - v;
}

// The bin where the descending cumulative count of the 4096-bin histogram h
// (shared memory) first reaches `need` (1 <= need <= sum h); *above = count in
// higher bins.  Thread t owns bins 4095-8t .. 4088-8t.
__device__ int find_threshold_bin(const uint32_t* h, uint32_t need, uint32_t* above) {
  static_assert(kSelThreads * 8 == kHistBins, "8 bins per thread");
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int top = kHistBins - 1 - 8 * int(threadIdx.x);
  uint32_t v[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = h[top - i];
    local += v[i];
  }
  const uint32_t excl = block_exclusive_scan(local, nullptr);
  if (excl < need && excl + local >= need) {
    uint32_t c = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (c < need && c + v[i] >= need) {
        s_bin = top - i;
        s_above = c;
      }
      c += v[i];
    }
  }
  __syncthreads();
  *above = s_above;
  const int r = s_bin;
  __syncthreads();
  return r;
}

template <typename T, bool ASC>
__device__ void bitonic_sort_smem(T* a, int n_pow2) {
  for (int size = 2; size <= n_pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = ((i & size) == 0) == ASC;
          const T x = a[i], y = a[j];
          if ((x > y) == up) {
            a[i] = y;
            a[j] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Ordered walk of a bitmap of `words` words: calls emit(index, rank) for
// every set bit in ascending index order (rank = 0, 1, ...).  Returns the count.
template <typename F>
__device__ uint32_t bitmap_ordered_walk(const uint32_t* bm, int words, F emit) {
  const int per = (words + kSelThreads - 1) / kSelThreads;
  const int w0 = min(words, int(threadIdx.x) * per), w1 = min(words, w0 + per);
  uint32_t local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(bm[w]);
  uint32_t total;
  uint32_t rank = block_exclusive_scan(local, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = bm[w];
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1;
      emit(uint32_t(w) * 32u + uint32_t(bit), rank++);
    }
  }
  return total;
}

// ------------------------------------------------------------------ filter + select
// Dynamic shared memory: two bitmaps of ceil(n/32) words when n <= kMaxBitmapN.
__global__ void __launch_bounds__(kSelThreads) index_filter_select(
    const float* __restrict__ scores, int64_t n, int k, int64_t chunk, uint32_t* __restrict__ hist,
    uint32_t* __restrict__ hist2, uint32_t* __restrict__ done, uint32_t* __restrict__ cand_count,
    uint64_t* __restrict__ cand, int64_t cap, int32_t* __restrict__ idx_out, int32_t* __restrict__ count_out,
    uint32_t* __restrict__ status) {
  extern __shared__ uint32_t dyn_bm[];
  __shared__ uint32_t sh[kHistBins];
  __shared__ int s_last;
  __shared__ uint32_t s_ntie, s_tie_min, s_tie_max, s_taken;
  __shared__ int32_t sel[2048];
  __shared__ uint64_t ties[kTieCap];

  const int b = blockIdx.y;
  const uint32_t kk = uint32_t(int64_t(k) < n ? int64_t(k) : n);
  uint32_t* hb = hist + size_t(b) * kHistBins;
  uint32_t* h2 = hist2 + size_t(b) * kHistBins;
  const float* sc = scores + size_t(b) * size_t(n);
  uint64_t* cb = cand + size_t(b) * size_t(cap);
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();

  // 1) threshold bin of the top-12-bit histogram
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = hb[i];
  __syncthreads();
  uint32_t above1;
  const int bin1 = find_threshold_bin(sh, kk, &above1);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0;
  __syncthreads();

  // 2) filter this CTA's chunk: candidates (bin >= bin1) and the next-12-bit
  //    histogram of the entries in bin1
  const int64_t n0 = int64_t(blockIdx.x) * chunk;
  const int64_t n1 = min(n, n0 + chunk);
  for (int64_t base = n0; base < n1; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    uint32_t o = 0;
    bool take = false;
    if (i < n1) {
      o = ord_f32(sc[i]);
      const int bin = int(o >> 20);
      take = bin >= bin1;
      if (bin == bin1) atomicAdd(&sh[(o >> 8) & 0xfffu], 1u);
    }
    const uint32_t m = __ballot_sync(kFull, take);
    if (m) {
      uint32_t pos0 = 0;
      if (lane == __ffs(m) - 1) pos0 = atomicAdd(&cand_count[b], uint32_t(__popc(m)));
      pos0 = __shfl_sync(kFull, pos0, __ffs(m) - 1);
      if (take) {
        const uint64_t pos = uint64_t(pos0) + __popc(m & ((1u << lane) - 1u));
        if (pos < uint64_t(cap)) cb[pos] = (uint64_t(o) << 32) | uint64_t(0xffffffffu - uint32_t(i));
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&h2[i], sh[i]);

  // 3) ticket: the last CTA of this sequence resolves the selection
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&done[b], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = __ldcg(&h2[i]);
  if (threadIdx.x == 0) {
    s_ntie = 0;
    s_tie_min = 0xffffffffu;
    s_tie_max = 0;
    s_taken = 0;
  }
  __syncthreads();
  uint32_t above2;
  const uint32_t need1 = kk - above1;  // still needed from bin1 (>= 1)
  const int bin2 = find_threshold_bin(sh, need1, &above2);
  const uint32_t prefix = (uint32_t(bin1) << 12) | uint32_t(bin2);  // 24-bit threshold prefix
  const uint32_t need_tie = need1 - above2;                           // >= 1
  const uint32_t total = __ldcg(&cand_count[b]);
  int32_t* ob = idx_out + size_t(b) * k;

  bool done_out = false;
  if (total <= uint64_t(cap) && n <= kMaxBitmapN) {
    // bitmap path: entries above the prefix into `selbm`, entries at the prefix into `tiebm`
    const int words = int((n + 31) / 32);
    uint32_t* selbm = dyn_bm;
    uint32_t* tiebm = dyn_bm + words;
    for (int w = threadIdx.x; w < 2 * words; w += blockDim.x) dyn_bm[w] = 0;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < total; c += blockDim.x) {
      const uint64_t key = __ldcg(&cb[c]);
      const uint32_t o = uint32_t(key >> 32), i = 0xffffffffu - uint32_t(key);
      const uint32_t pre = o >> 8;
      if (pre > prefix) {
        atomicOr(&selbm[i >> 5], 1u << (i & 31));
      } else if (pre == prefix) {
        atomicOr(&tiebm[i >> 5], 1u << (i & 31));
        atomicMin(&s_tie_min, o);
        atomicMax(&s_tie_max, o);
        const uint32_t slot = atomicAdd(&s_ntie, 1u);
        if (slot < kTieCap) ties[slot] = key;
      }
    }
    __syncthreads();
    const uint32_t n_tie = s_ntie;
    bool ties_ok = true;
    if (s_tie_min == s_tie_max) {
      // every entry at the prefix has the same score: the lowest indices win
      bitmap_ordered_walk(tiebm, words, [&](uint32_t i, uint32_t rank) {
        if (rank < need_tie) atomicOr(&selbm[i >> 5], 1u << (i & 31));
      });
    } else if (n_tie <= uint32_t(kTieCap)) {
      // distinct scores share the prefix: order those entries by (score desc, index asc)
      int np2 = 1;
      while (np2 < int(n_tie)) np2 <<= 1;
      for (int i = int(n_tie) + threadIdx.x; i < np2; i += blockDim.x) ties[i] = 0;
      __syncthreads();
      bitonic_sort_smem<uint64_t, false>(ties, np2);
      for (uint32_t t = threadIdx.x; t < need_tie; t += blockDim.x) {
        const uint32_t i = 0xffffffffu - uint32_t(ties[t]);
        atomicOr(&selbm[i >> 5], 1u << (i & 31));
      }
    } else {
      ties_ok = false;
    }
    __syncthreads();
    if (ties_ok) {
      const uint32_t got = bitmap_ordered_walk(selbm, words, [&](uint32_t i, uint32_t rank) {
        if (rank < kk) ob[rank] = int32_t(i);
      });
      if (threadIdx.x == 0 && got != kk) set_status(status, DSV4KV_DEV_INCONSISTENT);
      done_out = true;
    }
  }
  if (!done_out) {
    // General path (huge n, candidate overflow or massive heterogeneous ties):
    // exact threshold code o* from the low 8 bits of the entries at the
    // prefix, then one ordered scan over all scores keeps codes > o* and the
    // first r codes == o* (lowest indices).
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t o = ord_f32(sc[i]);
      if ((o >> 8) == prefix) atomicAdd(&sh[o & 0xffu], 1u);
    }
    __syncthreads();
    __shared__ uint32_t s_low, s_above3;
    if (threadIdx.x == 0) {
      uint32_t c = 0;
      for (int v = 255; v >= 0; --v) {
        if (c + sh[v] >= need_tie) {
          s_low = uint32_t(v);
          s_above3 = c;
          break;
        }
        c += sh[v];
      }
    }
    __syncthreads();
    const uint32_t ostar = (prefix << 8) | s_low;
    const uint32_t r_eq = need_tie - s_above3;  // entries equal to o* to keep
    __shared__ uint32_t s_gt_seen, s_eq_seen;
    if (threadIdx.x == 0) {
      s_gt_seen = 0;
      s_eq_seen = 0;
    }
    __syncthreads();
    for (int64_t base = 0; base < n; base += blockDim.x) {
      const int64_t i = base + threadIdx.x;
      const uint32_t o = i < n ? ord_f32(sc[i]) : 0u;
      const bool gt = i < n && o > ostar;
      const bool eq = i < n && o == ostar;
      uint32_t ngt, neq;
      const uint32_t gt_before = s_gt_seen + block_exclusive_scan(gt ? 1u : 0u, &ngt);
      const uint32_t eq_before = s_eq_seen + block_exclusive_scan(eq ? 1u : 0u, &neq);
      // index order is preserved: kept entries before this one = gt_before + min(eq_before, r_eq)
      const uint32_t pos = gt_before + min(eq_before, r_eq);
      if ((gt || (eq && eq_before < r_eq)) && pos < kk) ob[pos] = int32_t(i);
      if (threadIdx.x == 0) {
        s_gt_seen += ngt;
        s_eq_seen += neq;
      }
      __syncthreads();
    }
    if (threadIdx.x == 0 && s_gt_seen + min(s_eq_seen, r_eq) != kk) set_status(status, DSV4KV_DEV_INCONSISTENT);
  }
  for (int i = int(kk) + threadIdx.x; i < k; i += blockDim.x) ob[i] = -1;
  if (threadIdx.x == 0 && count_out) count_out[b] = int32_t(kk);

  // 4) leave the workspace zeroed for the next call
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    hb[i] = 0;
    h2[i] = 0;
  }
  if (threadIdx.x == 0) {
    cand_count[b] = 0;
    done[b] = 0;
  }
}

__global__ void index_fill_all(int64_t n, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ count_out) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < k; i += gridDim.x * blockDim.x)
    idx_out[size_t(b) * k + i] = i < n ? i : -1;
  if (count_out && blockIdx.x == 0 && threadIdx.x == 0) count_out[b] = int32_t(n);
}

// ------------------------------------------------------------------ host side
struct IndexWs {
  uint32_t* status;
  uint32_t* done;
  uint32_t* cand_count;
  uint32_t* hist;
  uint32_t* hist2;
  float* scores;
  uint64_t* cand;
  int64_t cap;
  size_t bytes;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static IndexWs index_ws_layout(char* base, int batch, int64_t n, int k) {
  IndexWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  };
  w.status = reinterpret_cast<uint32_t*>(take(16));
  w.done = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * batch));
  w.cand_count = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * batch));
  w.hist = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * kHistBins * size_t(batch)));
  w.hist2 = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * kHistBins * size_t(batch)));
  w.scores = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * size_t(n)));
  w.cap = std::max<int64_t>(8192, 2 * int64_t(k));
  w.cand = reinterpret_cast<uint64_t*>(take(sizeof(uint64_t) * size_t(batch) * size_t(w.cap)));
  w.bytes = off;
  return w;
}

size_t index_topk_ws_bytes(int batch, int64_t n, int k) { return index_ws_layout(nullptr, batch, n, k).bytes; }

// Bytes at the start of the workspace that must be zero before a call (status
// word, counters, histograms): everything before the scores.
size_t index_topk_zero_prefix_bytes(int batch) {
  const IndexWs w = index_ws_layout(nullptr, batch, 1, 1);
  return size_t(reinterpret_cast<char*>(w.scores) - static_cast<char*>(nullptr));
}

dsv4kv_status index_topk_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n, int k,
                                int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  if (n <= k) {
    const dim3 grid((unsigned)((k + 255) / 256), (unsigned)batch);
    if (launch_pdl(index_fill_all, grid, dim3(256), 0, stream, n, k, idx_out, count_out) != cudaSuccess)
      return check_launch("index_fill_all");
    return check_launch("index_fill_all");
  }
  const IndexWs w = index_ws_layout(static_cast<char*>(ws), batch, n, k);
  if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "index_topk: workspace too small");
  const int sms = sm_count();
  if (keys.fmt == DSV4KV_BF16) {
    // one wave (resident CTAs per SM x SMs) over the flattened (sequence, entry) range
    static int occ = 0;
    if (occ == 0 &&
        (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, index_score_bf16<8, true>, 256, 0) != cudaSuccess ||
         occ < 1))
      occ = 1;
    const int64_t total = int64_t(batch) * n;
    const int64_t grid = int64_t(sms) * occ;
    const int64_t per_cta = std::max<int64_t>(64, (total + grid - 1) / grid);
    launch_pdl(index_score_bf16<8, true>, dim3(unsigned((total + per_cta - 1) / per_cta)), dim3(256), 0, stream, qidx,
               static_cast<const uint16_t*>(keys.codes), keys.rows, n, batch, per_cta, w.scores, w.hist);
  } else {
    const int64_t target = int64_t(sms) * 4;
    int64_t splits = std::max<int64_t>(1, (target + batch - 1) / batch);
    int64_t chunk = (n + splits - 1) / splits;
    chunk = std::max<int64_t>(256, (chunk + 31) / 32 * 32);
    splits = (n + chunk - 1) / chunk;
    const dim3 g1((unsigned)splits, (unsigned)batch);
    launch_pdl(index_score_fp4, g1, dim3(256), 0, stream, qidx, static_cast<const uint8_t*>(keys.codes),
               static_cast<const uint8_t*>(keys.scales), keys.rows, n, chunk, w.scores, w.hist);
  }
  dsv4kv_status st = check_launch("index_score");
  if (st != DSV4KV_OK) return st;
  // filter/select: chunks of 4096 scores
  int64_t chunk2 = 4096;
  int64_t splits2 = (n + chunk2 - 1) / chunk2;
  const dim3 g2((unsigned)splits2, (unsigned)batch);
  const size_t dyn = n <= kMaxBitmapN ? size_t(2) * size_t((n + 31) / 32) * sizeof(uint32_t) : 0;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(index_filter_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(2 * (kMaxBitmapN / 32) * sizeof(uint32_t))) != cudaSuccess)
      return check_launch("index_filter_select: cudaFuncSetAttribute");
    attr_set = true;
  }
  launch_pdl(index_filter_select, g2, dim3(kSelThreads), dyn, stream, w.scores, n, k, chunk2, w.hist, w.hist2, w.done,
             w.cand_count, w.cand, w.cap, idx_out, count_out, w.status);
  return check_launch("index_filter_select");
}

}  // namespace dsv4kv
