// Lightning indexer scores and exact top-k selection.
//
// [P1] "c4a (the milder scheme)": DeepSeek Sparse Attention keeps the top-k
// (k = 512) compressed entries per query; [P1] indexer paragraph: the indexer
// cache holds 128 values per entry and may be fp4; [P2] Step 5: the learned
// indexer scores compressed blocks and the query reads the selected ones.
//
// Two launches per call (both on the caller's stream):
//  1. index_score_*: streams the keys once (bulk copies into shared memory,
//     half a warp per bf16 key; 16-byte vector loads, a quarter warp per fp4
//     key), writes one fp32 score per
//     entry to the workspace and builds a per-sequence histogram of the top
//     12 bits of the order-preserving score code.
//  2. index_select: several CTAs per sequence filter the scores against the
//     threshold bin of that histogram into a candidate list; the first of
//     them resolves the exact selection from the candidates (two more
//     histogram levels down to the exact threshold code, the lowest indices
//     among equal scores, index-ordered output) and the sequence's histogram
//     is re-zeroed.
//  (only when n <= k) index_fill_all writes 0..n-1 directly.
// The order (score desc, index asc) is a total order, so the result is the
// same for every split of the entries (exact, not approximate).
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

constexpr int kHistBins = 4096;  // 12-bit digits

// The global histograms keep bin i at position ((i & 31) << 7) | (i >> 5):
// neighbouring bins sit 512 bytes apart, in different L2 lines.  Most scores
// fall into a few neighbouring bins, and with many CTAs adding into one
// sequence's histogram (small batches), atomics that all hit the same few
// lines would queue behind each other.
__host__ __device__ __forceinline__ int hist_pos(int bin) { return ((bin & 31) << 7) | (bin >> 5); }
__host__ __device__ __forceinline__ int hist_bin(int pos) { return ((pos & 127) << 5) | (pos >> 7); }

// Row stride of the fp32 score rows in the workspace: n rounded up to 4, so
// every row starts on a 16-byte boundary.
__host__ __device__ __forceinline__ int64_t score_stride(int64_t n) { return (n + 3) & ~int64_t(3); }

// ------------------------------------------------------------------ scoring
// Transposing butterfly: lane l16 of a 16-lane group holds U partial sums
// (one per key); after log2 steps each lane holds the full 16-lane sum of one
// key.  U = 16: key l16 (15 shuffles for 16 keys).  U = 8: key (l16 >> 1) & 7,
// duplicated on lanes 2i and 2i+1 (8 shuffles for 8 keys).  U = 4: key
// (l16 >> 2) & 3 on lanes 4i..4i+3 (4 shuffles for 4 keys).
template <int U>
__device__ __forceinline__ float reduce16_transposed(const float (&p)[U], int l16) {
  if constexpr (U == 4) {
    const bool b3 = l16 & 8, b2 = l16 & 4;
    float c[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) c[i] = (b3 ? p[2 + i] : p[i]) + __shfl_xor_sync(kFull, b3 ? p[i] : p[2 + i], 8);
    float s = (b2 ? c[1] : c[0]) + __shfl_xor_sync(kFull, b2 ? c[0] : c[1], 4);
    s += __shfl_xor_sync(kFull, s, 2);
    return s + __shfl_xor_sync(kFull, s, 1);
  }
  static_assert(U == 8 || U == 16 || U == 4, "keys per half-warp");
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

// Adds the CTA's histogram sh to the sequence's global histogram and clears it.
__device__ __forceinline__ void flush_histogram(uint32_t* sh, uint32_t* hb) {
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    const uint32_t c = sh[i];
    if (c) {
      atomicAdd(&hb[hist_pos(i)], c);
      sh[i] = 0;
    }
  }
}

// Share of every sequence's keys scored from the shared queue of the bf16
// score kernel, and the smallest batch that uses it.
constexpr int kTailPct = 25;
constexpr int kTailMinBatch = 16;

// The four code bytes of w (byte 0 = lowest) decoded to four f16x2 pairs by
// cvt.rn.f16x2.e2m1x2 straight from the unpacked bytes (no shifts or masks);
// each pair holds (low nibble, high nibble) = (even, odd) channel.
__device__ __forceinline__ void e2m1x8_unpack(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// sum_g scale_g * (even_g + odd_g) over the two 16-channel groups of a lane:
// acc0 / acc1 are the f16x2 (even, odd) channel sums of groups 0 / 1 and s2
// their two E4M3 scale bytes (group 0 in the low byte).  The halves are added
// in f16 (exact while the sums are multiples of 0.5 below 1024, as for the
// integer-valued keys of the indexer), the scales converted by one cvt, the
// products taken in fp32.
__device__ __forceinline__ float scaled_group_sums(uint32_t acc0, uint32_t acc1, uint32_t s2) {
  uint32_t ev, od, t, sc;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(ev) : "r"(acc0), "r"(acc1));  // (even0, even1)
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(od) : "r"(acc0), "r"(acc1));  // (odd0, odd1)
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(ev), "r"(od));
  asm("{\n\t.reg .b16 b;\n\tcvt.u16.u32 b, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, b;\n\t}" : "=r"(sc) : "r"(s2));
  float t0, t1, s0, s1;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(t0), "=f"(t1) : "r"(t));
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(s0), "=f"(s1) : "r"(sc));
  return fmaf(t1, s1, t0 * s0);
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}

// fp4 keys, dim 128: 64 B of codes + 8 E4M3 scale bytes per key.  A quarter
// warp (4 lanes x 16 B) covers one key; lane l4 holds channels
// [32*l4, 32*l4+32) = two 16-channel scale groups; a warp takes 32 keys (4
// per quad).  Each code byte is decoded to a packed f16 pair with
// cvt.rn.f16x2.e2m1x2 and accumulated with packed f16 FMAs per group (exact
// for integer queries: |partial| <= 8*8*6 per half at a resolution of 0.5),
// then scaled by the group's E4M3 scale in fp32 (StreamConsumer<StreamFp4>).

// index_score_stream<F>: the score kernel with the keys streamed into shared
// memory by bulk copies.  One CTA per SM: a producer thread (the last warp)
// feeds a ring of F::kStages stages of up to F::kKeys keys (codes, the fp4
// keys' group scales, and the sequence's query), each completing on its own
// mbarrier; F::kConsumers consumer warps score every stage and free it as
// soon as its keys are in their registers.  The producer walks the CTA's
// even share of the first n_h keys of every sequence (flattened over the
// batch; stages never straddle two sequences), then claims F::kKeys-key
// units of the sequences' tails from the shared counter (batches of
// kTailMinBatch or more), so the CTAs that stream faster take more of the
// tail.  Histogram counts of the even share go to one of two shared-memory
// histograms (the CTA's first two sequences; an even share spans at most two
// when it is shorter than n_h) flushed once at the end; tail counts and
// those of further sequences go straight to global memory.  Every wait is
// bounded; a wait that gives up flags DSV4KV_DEV_TIMEOUT and ends the loop.
//
// bf16 keys: 128 keys (32 KB) per stage, 8 consumer warps, a warp 16 keys,
// half a warp per key (as the bf16 scoring elsewhere in this file).  fp4
// keys: 512 keys (32 KB of codes + 4 KB of scales) per stage, 16 consumer
// warps, a warp 32 keys, a quarter warp per key (see the fp4 note above).
struct StreamBf16 {
  static constexpr int kKeys = 128, kConsumers = 8, kStages = 5;
  static constexpr uint32_t kCodeBytes = 256, kScaleBytes = 0;  // per key
};
struct StreamFp4 {
  static constexpr int kKeys = 512, kConsumers = 16, kStages = 5;
  static constexpr uint32_t kCodeBytes = 64, kScaleBytes = 8;
};
template <class F>
struct StreamLayout {
  static constexpr uint32_t kCodes = F::kKeys * F::kCodeBytes;
  // the scale rows are copied from an even row on (a bulk copy moves whole
  // 16-byte units), so a stage holds up to two more of them
  static constexpr uint32_t kScales = F::kScaleBytes ? (F::kKeys + 2) * F::kScaleBytes : 0;
  static constexpr uint32_t kStage = kCodes + kScales + 256;  // codes, scales, the query
  static constexpr int kThreads = 32 * (F::kConsumers + 1);
};
struct StreamMeta {
  int32_t b, cnt;  // cnt < 0: no more stages
  int64_t i0;
  int32_t tail;
  int32_t soff;  // key 0's row among the stage's scale rows (0 or 1)
};
template <class F>
struct StreamCtl {
  uint64_t full[F::kStages];
  uint64_t empty[F::kStages];
  StreamMeta meta[F::kStages];
  int abort;
};
template <class F>
constexpr size_t stream_smem() {
  return size_t(F::kStages) * StreamLayout<F>::kStage + 2 * kHistBins * sizeof(uint32_t) + sizeof(StreamCtl<F>) + 128;
}
static_assert(stream_smem<StreamBf16>() <= 232448 && stream_smem<StreamFp4>() <= 232448, "shared memory per CTA");
constexpr uint64_t kStreamWaitNs = 1000000000ull;

__device__ __forceinline__ uint64_t stream_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait on one phase of an mbarrier (the calling thread polls).
template <class F>
__device__ __forceinline__ bool stream_wait(uint64_t* bar, uint32_t parity, StreamCtl<F>* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = stream_now();
  while (!mbar_try_wait(bar, parity)) {
    if (ctl->abort || stream_now() - t0 > kStreamWaitNs) {
      ctl->abort = 1;
      return false;
    }
  }
  return true;
}

// Where a consumer finds what a stage does not hold: the scale row of the
// last key row when the rows total is odd (bulk copies move whole 16-byte
// units, two scale rows).
struct StreamEdge {
  const uint8_t* scales;
  int64_t key_rows, last_odd_row;  // last_odd_row < 0: none
};

// A consumer warp's part of one stage: load() brings the warp's keys and the
// query into registers (after it the stage may be refilled); score() leaves
// on each lane the score of key `key` of the stage, to be stored by the
// lanes with `writer` set.
template <class F>
struct StreamConsumer;

template <>
struct StreamConsumer<StreamBf16> {
  uint4 v[8];
  float q[8];
  __device__ __forceinline__ void load(const uint8_t* st, const StreamMeta&, const StreamEdge&, int warp, int lane) {
    const int half = lane >> 4, l16 = lane & 15;
    const uint4 x = *reinterpret_cast<const uint4*>(st + StreamLayout<StreamBf16>::kCodes + 16 * l16);
    q[0] = bf16lo(x.x); q[1] = bf16hi(x.x); q[2] = bf16lo(x.y); q[3] = bf16hi(x.y);
    q[4] = bf16lo(x.z); q[5] = bf16hi(x.z); q[6] = bf16lo(x.w); q[7] = bf16hi(x.w);
    const int k0 = 16 * warp + 8 * half;  // this half-warp's first key of the stage
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = *reinterpret_cast<const uint4*>(st + (k0 + u) * 256 + 16 * l16);
  }
  __device__ __forceinline__ float score(int warp, int lane, int* key, bool* writer) const {
    const int half = lane >> 4, l16 = lane & 15;
    float p[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) p[u] = dot8_bf16(v[u], q);  // (keys past cnt: stale data, never stored)
    *key = 16 * warp + 8 * half + ((l16 >> 1) & 7);  // reduce16_transposed<8>: lanes 2i, 2i+1 hold key i
    *writer = !(lane & 1);
    return reduce16_transposed<8>(p, l16) + 0.0f;  // -0 -> +0
  }
};

template <>
struct StreamConsumer<StreamFp4> {
  uint4 v[4];
  uint32_t s2[4];
  uint32_t qp[16];  // (q[2j], q[2j+1]) as f16x2 for this lane's 32 channels
  __device__ __forceinline__ void load(const uint8_t* st, const StreamMeta& m, const StreamEdge& e, int warp,
                                       int lane) {
    using Lay = StreamLayout<StreamFp4>;
    const int quad = lane >> 2, l4 = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x = *reinterpret_cast<const uint4*>(st + Lay::kCodes + Lay::kScales + 64 * l4 + 16 * i);
      qp[4 * i] = f32x2_to_f16x2(bf16lo(x.x), bf16hi(x.x));
      qp[4 * i + 1] = f32x2_to_f16x2(bf16lo(x.y), bf16hi(x.y));
      qp[4 * i + 2] = f32x2_to_f16x2(bf16lo(x.z), bf16hi(x.z));
      qp[4 * i + 3] = f32x2_to_f16x2(bf16lo(x.w), bf16hi(x.w));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int key = 32 * warp + 8 * u + quad;
      v[u] = *reinterpret_cast<const uint4*>(st + key * 64 + 16 * l4);
      const int64_t row = int64_t(m.b) * e.key_rows + m.i0 + key;
      s2[u] = row == e.last_odd_row && key < m.cnt
                  ? uint32_t(*reinterpret_cast<const uint16_t*>(e.scales + row * 8 + 2 * l4))
                  : uint32_t(*reinterpret_cast<const uint16_t*>(st + Lay::kCodes + (m.soff + key) * 8 + 2 * l4));
    }
  }
  __device__ __forceinline__ float score(int warp, int lane, int* key, bool* writer) const {
    const int quad = lane >> 2, l4 = lane & 3;
    float p[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t acc0 = 0, acc1 = 0;  // f16x2 sums of group 0 (words 0, 1) and group 1 (words 2, 3)
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        uint32_t h[4];
        e2m1x8_unpack(w[wi], h);
#pragma unroll
        for (int by = 0; by < 4; ++by) {
          if (wi < 2) acc0 = hfma2(qp[4 * wi + by], h[by], acc0);
          else acc1 = hfma2(qp[4 * wi + by], h[by], acc1);
        }
      }
      p[u] = scaled_group_sums(acc0, acc1, s2[u]);
    }
    // reduce over the 4 lanes of the quad: 4 values -> transposing butterfly
    const bool bb1 = l4 & 2, bb0 = l4 & 1;
    float k2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) k2[i] = (bb1 ? p[2 + i] : p[i]) + __shfl_xor_sync(kFull, bb1 ? p[i] : p[2 + i], 2);
    *key = 32 * warp + 8 * l4 + quad;  // lane l4 ends with key u = l4
    *writer = true;
    return (bb0 ? k2[1] : k2[0]) + __shfl_xor_sync(kFull, bb0 ? k2[0] : k2[1], 1) + 0.0f;
  }
};

template <class F>
__global__ void __launch_bounds__(StreamLayout<F>::kThreads, 1)
    index_score_stream(const uint16_t* __restrict__ qidx, const uint8_t* __restrict__ codes,
                       const uint8_t* __restrict__ scales, int64_t key_rows, int64_t n, int64_t n_h, int batch,
                       int64_t per_cta, float* __restrict__ scores, uint32_t* __restrict__ hist,
                       uint32_t* __restrict__ tail_ctr, uint32_t* __restrict__ status) {
  using Lay = StreamLayout<F>;
  constexpr int S = F::kStages;
  extern __shared__ __align__(128) uint8_t sraw[];
  uint8_t* stage = sraw;
  uint32_t* sh = reinterpret_cast<uint32_t*>(sraw + size_t(S) * Lay::kStage);  // [2][kHistBins]
  StreamCtl<F>* ctl = reinterpret_cast<StreamCtl<F>*>(sh + 2 * kHistBins);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], F::kConsumers);
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * kHistBins; i += Lay::kThreads) sh[i] = 0;
  __syncthreads();
  pdl_wait();
  const int64_t total = int64_t(batch) * n_h;
  const int64_t g0 = min(total, int64_t(blockIdx.x) * per_cta), g1 = min(total, g0 + per_cta);
  const int64_t tups = (n - n_h + F::kKeys - 1) / F::kKeys;  // tail units per sequence
  const int64_t rows_total = int64_t(batch) * key_rows;      // rows of the key (and scale) arrays
  const int64_t TU = n_h < n ? int64_t(batch) * tups : 0;

  if (warp == F::kConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();  // keys are read once
      int64_t pos = g0;
      uint32_t claimed = TU > 0 ? atomicAdd(tail_ctr, 1u) : 0u;  // one claim ahead
      int it = 0;
      bool ok = true;
      for (;; ++it) {
        int b, cnt, tail;
        int64_t i0;
        if (pos < g1) {
          b = int(pos / n_h);
          i0 = pos - int64_t(b) * n_h;
          const int64_t end = min(g1, int64_t(b + 1) * n_h);
          cnt = int(min(int64_t(F::kKeys), end - pos));
          pos += cnt;
          tail = 0;
        } else if (int64_t(claimed) < TU) {
          b = int(int64_t(claimed) / tups);
          i0 = n_h + (int64_t(claimed) % tups) * F::kKeys;
          cnt = int(min(int64_t(F::kKeys), n - i0));
          tail = 1;
          claimed = atomicAdd(tail_ctr, 1u);
        } else {
          break;
        }
        const int s = it % S;
        if (it >= S && !stream_wait(&ctl->empty[s], ((it / S) - 1) & 1, ctl)) {
          ok = false;
          break;
        }
        uint8_t* dst = stage + size_t(s) * Lay::kStage;
        const int64_t row = int64_t(b) * key_rows + i0;
        const uint32_t cbytes = uint32_t(cnt) * F::kCodeBytes;
        // scale rows [r0, r1): from the even row at or below the first key to
        // the even row at or above the end, but never past the last even row
        // of the array (an odd total's last row is read by the consumers)
        int64_t r0 = row, r1 = row;
        if constexpr (F::kScaleBytes > 0) {
          r0 = row & ~int64_t(1);
          r1 = min((row + cnt + 1) & ~int64_t(1), rows_total & ~int64_t(1));
        }
        const uint32_t sbytes = uint32_t(r1 - r0) * F::kScaleBytes;
        ctl->meta[s] = StreamMeta{b, cnt, i0, tail, int32_t(row - r0)};
        mbar_arrive_expect_tx(&ctl->full[s], cbytes + sbytes + 256u);
        bulk_load(dst, codes + size_t(row) * F::kCodeBytes, cbytes, &ctl->full[s], pol);
        if (sbytes > 0) bulk_load(dst + Lay::kCodes, scales + size_t(r0) * F::kScaleBytes, sbytes, &ctl->full[s], pol);
        bulk_load_plain(dst + Lay::kCodes + Lay::kScales, qidx + size_t(b) * 128, 256u, &ctl->full[s]);
      }
      bool marked = false;
      if (ok) {  // the end marker
        const int s = it % S;
        if (it < S || stream_wait(&ctl->empty[s], ((it / S) - 1) & 1, ctl)) {
          ctl->meta[s] = StreamMeta{0, -1, 0, 0, 0};
          mbar_arrive(&ctl->full[s]);
          marked = true;
        }
      }
      // Normally the consumers wait for every copy before they finish.  After
      // a wait that gave up, never leave with copies in flight: wait (bounded)
      // for the last phase of each stage still armed (none was re-armed by a
      // marker on this path).
      if (!marked) {
        const uint64_t t0 = stream_now();
        for (int j = max(0, it - S); j < it; ++j)
          while (!mbar_try_wait(&ctl->full[j % S], (j / S) & 1))
            if (stream_now() - t0 > kStreamWaitNs) break;
      }
      if (ctl->abort) set_status(status, DSV4KV_DEV_TIMEOUT);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int b0 = n_h > 0 ? int(g0 / n_h) : 0;  // the even share's first sequence: shared histogram 0
  const StreamEdge edge{scales, key_rows, (rows_total & 1) ? rows_total - 1 : -1};
  for (int it = 0;; ++it) {
    const int s = it % S;
    bool ok = true;
    if (lane == 0) ok = stream_wait(&ctl->full[s], (it / S) & 1, ctl);
    if (!__shfl_sync(kFull, ok, 0)) break;
    const StreamMeta m = ctl->meta[s];
    if (m.cnt < 0) break;
    StreamConsumer<F> c;
    c.load(stage + size_t(s) * Lay::kStage, m, edge, warp, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->empty[s]);  // the warp's keys are in registers
    int key;
    bool writer;
    const float sc = c.score(warp, lane, &key, &writer);
    if (writer && key < m.cnt) {
      scores[size_t(m.b) * size_t(score_stride(n)) + size_t(m.i0 + key)] = sc;
      const int bin = int(ord_f32(sc) >> 20), slot = m.b - b0;
      if (!m.tail && slot >= 0 && slot < 2) atomicAdd(&sh[slot * kHistBins + bin], 1u);
      else atomicAdd(&hist[size_t(m.b) * kHistBins + hist_pos(bin)], 1u);
    }
  }
  // flush the two shared histograms (every consumer warp ends its loop: the waits are bounded)
  asm volatile("barrier.cta.sync 1, %0;" ::"n"(32 * F::kConsumers) : "memory");
  for (int i = threadIdx.x; i < 2 * kHistBins; i += 32 * F::kConsumers) {
    const uint32_t c = sh[i];
    const int bb = b0 + i / kHistBins;
    if (c && bb < batch) atomicAdd(&hist[size_t(bb) * kHistBins + hist_pos(i % kHistBins)], c);
  }
}

// ------------------------------------------------------------------ selection
// index_select runs one thread-block cluster of C CTAs per sequence (grid
// C x B).  Every CTA finds the threshold bin b1 of its sequence in the score
// kernel's histogram and filters its chunk of scores (the loads of a batch in
// flight before any is inspected) into a shared-memory list of candidates
// (top-12-bit bin >= b1), kept in index order.  After a cluster barrier the
// leader CTA reads every CTA's list through distributed shared memory, in
// chunk order, so the candidates arrive sorted by index; the other CTAs wait
// at a second barrier until it has, then exit.  The leader resolves the exact
// selection from the candidates alone: the histogram of bits 8-19 of the
// codes in b1 gives the 24-bit threshold prefix, the histogram of bits 0-7 of
// the codes at that prefix the exact threshold code T; every code above T is
// in, and of the codes equal to T (equal scores) the earliest positions
// (lowest indices) fill what is missing, found by an ordered scan; an ordered
// compaction writes the result in ascending index order.  The sequence's
// histogram is re-zeroed for the next call.
constexpr int kSelThreads = 512;
constexpr int kSelBatch = 8;                           // scores per lane and warp batch
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelWarpSpan = 32 * kSelBatch;           // 256 scores per warp batch
constexpr int kSelChunkUnit = 4096;                    // CTA chunks are multiples of this
constexpr int kSelStage = 4096;                        // candidates a CTA can hold
// candidates per sequence the leader resolves in registers (4 per thread):
// the scores at or above the threshold bin, a few hundred for the c4a
// workloads; more (heavy ties) take the exact fallback scan.  A larger cap
// unrolls the leader's loops further, and the instruction-cache misses of
// that code cost more than the rare fallback saves (16 per thread: the
// selection 17.3 -> 14.3 us per call at B = 32).
constexpr int kCandCap = 2048;
// entries of the leader's receive buffer: CTA r of a C-CTA cluster pushes its
// list into region r (kRecvCap / C entries), so the candidates of one part of
// a sequence (scores that cluster by position) fit as well as spread ones
constexpr int kRecvCap = 8192;
constexpr int kResPer = kCandCap / kSelThreads;        // candidates per leader thread
constexpr int kMaxClusterSel = 16;
constexpr int kWarpCap = kSelStage / kSelWarps;       // candidates a warp's list can hold
// Every warp streams its run of scores through its own ring of kRing slots
// of one warp batch (256 fp32 = 1 KB) in shared memory, filled by 16-byte
// cp.async copies kRing - 1 batches ahead of the one it filters.
constexpr int kRing = 4;
constexpr size_t kRingBytes = size_t(kSelWarps) * kRing * kSelWarpSpan * sizeof(float);  // 64 KB
// dynamic shared memory: the rings, the warps' lists (kSelStage u64), and the
// leader's receive buffer (kRecvCap u64)
constexpr size_t kSelDyn = kRingBytes + (size_t(kSelStage) + kRecvCap) * sizeof(uint64_t);

// Block-wide exclusive prefix sum of one value per thread (NT threads).
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* total) {
  __shared__ uint32_t wsum[NT / 32];
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
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t x = wsum[w];
    base += w < warp ? x : 0u;
    all += x;
  }
  __syncthreads();
  if (total) *total = all;
  return base + incl - v;
}

__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Adds 1 to bin `bin` of the shared histogram h for every active lane, one
// atomic per distinct bin of the warp: lanes with equal bins (common when
// many scores are equal) are counted by their lowest lane.
__device__ __forceinline__ void hist_add_warp(uint32_t* h, bool active, uint32_t bin) {
  if (!__any_sync(kFull, active)) return;
  const uint32_t peers = __match_any_sync(kFull, active ? bin : 0xffffffffu);
  if (active && __ffs(peers) - 1 == int(threadIdx.x & 31)) atomicAdd(&h[bin], uint32_t(__popc(peers)));
}

// The bin where the descending cumulative count of the 4096-bin histogram h
// (shared memory, 16-byte aligned) first reaches `need` (1 <= need <= sum h);
// *above = count in higher bins.  Warp w owns the S = 4096/warps highest bins
// below those of warp w-1; lane l of it owns a contiguous run of PER = S/32
// bins (highest run on lane 0), read with 16-byte loads.  One warp scan over
// the lanes' run sums finds the crossing lane, which walks its own run.
template <int NT>
__device__ int find_threshold_bin(const uint32_t* h, uint32_t need, uint32_t* above) {
  constexpr int NW = NT / 32, SPAN = kHistBins / NW, PER = SPAN / 32;
  static_assert(PER % 4 == 0 && PER * 32 * NW == kHistBins, "bins per lane");
  __shared__ uint32_t s_wtot[NW];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lo = kHistBins - SPAN * warp - PER * (lane + 1);  // lowest bin of this lane's run
  uint32_t v[PER], sum = 0;
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const uint4 x = *reinterpret_cast<const uint4*>(h + lo + 4 * q);
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) sum += v[i];
  const uint32_t incl = warp_inclusive_scan(sum);  // lane order = descending bins
  if (lane == 31) s_wtot[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) before += w < warp ? s_wtot[w] : 0u;  // independent loads, no chain
  const uint32_t ex = before + incl - sum;  // entries in higher bins than this run
  if (ex < need && ex + sum >= need) {      // exactly one lane: walk its run from the top
    uint32_t c = ex;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (c < need && c + v[i] >= need) {
        s_bin = lo + i;
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

// Ordered compaction offsets for BATCH elements per thread at positions
// (j, warp, lane) in that lexicographic order: m[j] is the warp's ballot of
// the predicate for element j; off[j] receives the number of true elements
// before lane 0 of (j, warp).  Returns the total.  Block-wide (syncs).
template <int NT, int BATCH>
__device__ uint32_t ordered_offsets(const uint32_t (&m)[BATCH], uint32_t (&off)[BATCH]) {
  constexpr int NW = NT / 32, E = BATCH * NW, PER = E / 32;
  static_assert(PER * 32 == E, "entries per lane");
  __shared__ uint32_t s_c[E];
  __shared__ uint32_t s_total;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < BATCH; ++j) s_c[j * NW + warp] = __popc(m[j]);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x[PER], loc = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      x[q] = s_c[PER * lane + q];
      loc += x[q];
    }
    const uint32_t incl = warp_inclusive_scan(loc);
    uint32_t run = incl - loc;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      s_c[PER * lane + q] = run;
      run += x[q];
    }
    if (lane == 31) s_total = incl;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < BATCH; ++j) off[j] = s_c[j * NW + warp];
  const uint32_t total = s_total;
  __syncthreads();  // s_c is rewritten by the next call
  return total;
}

// ordered_offsets for two predicates at once: off[j] receives (count of a
// before lane 0 of (j, warp)) << 16 | (count of e before it); returns the
// totals packed the same way.  Every count must stay below 2^16.
template <int NT, int BATCH>
__device__ uint32_t ordered_offsets_pair(const uint32_t (&a)[BATCH], const uint32_t (&e)[BATCH],
                                         uint32_t (&off)[BATCH]) {
  constexpr int NW = NT / 32, E = BATCH * NW, PER = E / 32;
  static_assert(PER * 32 == E, "entries per lane");
  __shared__ uint32_t s_c[E];
  __shared__ uint32_t s_total;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < BATCH; ++j) s_c[j * NW + warp] = (uint32_t(__popc(a[j])) << 16) | uint32_t(__popc(e[j]));
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x[PER], loc = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      x[q] = s_c[PER * lane + q];
      loc += x[q];
    }
    const uint32_t incl = warp_inclusive_scan(loc);
    uint32_t run = incl - loc;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      s_c[PER * lane + q] = run;
      run += x[q];
    }
    if (lane == 31) s_total = incl;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < BATCH; ++j) off[j] = s_c[j * NW + warp];
  const uint32_t total = s_total;
  __syncthreads();  // s_c is rewritten by the next call
  return total;
}

// Copies a sequence's 4096-bin histogram from the workspace (L2) into shared
// memory in bin order: fetch() issues a thread's loads, store() writes them.
// Lane l of warp w takes the 16-byte group q = 32 l + (w + j NW) of
// positions (iteration j): the four bins of a group are 32 apart and the
// lanes' bins fall in 32 different banks.
template <int NT>
struct HistLoad {
  static constexpr int NW = NT / 32, V = 32 / NW;  // uint4 per thread
  static_assert(V * NW == 32 && V * 4 * NT == kHistBins, "histogram split");
  uint4 v[V];
  // the loads (issued before anything else the thread asks of memory)
  __device__ __forceinline__ void fetch(const uint32_t* __restrict__ hb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int j = 0; j < V; ++j) v[j] = __ldcg(reinterpret_cast<const uint4*>(hb) + 32 * lane + warp + j * NW);
  }
  __device__ __forceinline__ void store(uint32_t* sh) const;
};
template <int NT>
__device__ __forceinline__ void HistLoad<NT>::store(uint32_t* sh) const {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int p = 4 * (32 * lane + warp + j * NW);  // positions p .. p + 3
    sh[hist_bin(p)] = v[j].x;
    sh[hist_bin(p + 1)] = v[j].y;
    sh[hist_bin(p + 2)] = v[j].z;
    sh[hist_bin(p + 3)] = v[j].w;
  }
}

// Issues the copy of one warp batch (scores [base, base + 256) of the row,
// those at or beyond `end` zero-filled and not read) into a ring slot: lane l
// copies 16-byte pieces l and l + 32.  base is a multiple of 32 and the row
// 16-byte aligned, so every piece is aligned.
__device__ __forceinline__ void warp_issue_batch(const float* __restrict__ sc, int64_t base, int64_t end,
                                                 float* slot) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int piece = lane + 32 * h;
    const int64_t i = base + 4 * piece;
    const int64_t left = end - i;
    const uint32_t bytes = left >= 4 ? 16u : (left > 0 ? uint32_t(left) * 4u : 0u);
    cp_async16_zfill(slot + 4 * piece, bytes ? sc + i : sc, bytes);
  }
}

// The codes of a landed warp batch: lane l takes positions 32 v + l.
__device__ __forceinline__ void warp_read_batch(const float* slot, uint32_t (&o)[kSelBatch]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int v = 0; v < kSelBatch; ++v) o[v] = ord_f32(slot[32 * v + lane]);
}

// Appends, in index order, the warp batch's entries whose top-12-bit bin is
// >= bin1 to the warp's list (u64 = code << 32 | ~index) after `count`
// entries; returns the new count (entries beyond kWarpCap are counted, not
// stored).  Warp-synchronous: ballots give the order, no block barrier.
__device__ __forceinline__ uint32_t warp_stage_batch(const uint32_t (&o)[kSelBatch], int64_t base, int64_t end,
                                                     int bin1, uint32_t count, uint64_t* list) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int v = 0; v < kSelBatch; ++v) {
    const int64_t i = base + 32 * v + lane;
    const bool keep = i < end && int(o[v] >> 20) >= bin1;
    const uint32_t m = __ballot_sync(kFull, keep);
    if (keep) {
      const uint32_t at = count + __popc(m & lt);
      if (at < uint32_t(kWarpCap)) list[at] = (uint64_t(o[v]) << 32) | uint64_t(0xffffffffu - uint32_t(i));
    }
    count += __popc(m);
  }
  return count;
}

// Exact selection with no candidate list (the candidates overflowed the
// leader's buffer): the threshold code o* from the low 8 bits of the
// entries at the 24-bit prefix, then one ordered scan of all scores keeps
// codes > o* and the first r codes == o* (the lowest indices), in index order.
template <int NT>
__device__ void select_by_scan(const float* __restrict__ sc, int64_t n, uint32_t prefix, uint32_t need_tie,
                               uint32_t kk, int32_t* __restrict__ ob, uint32_t* sh256, uint32_t* status) {
  __shared__ uint32_t s_low, s_above3, s_gt_seen, s_eq_seen;
  for (int i = threadIdx.x; i < 256; i += NT) sh256[i] = 0;
  __syncthreads();
  for (int64_t i = threadIdx.x; i < n; i += NT) {
    const uint32_t o = ord_f32(sc[i]);
    if ((o >> 8) == prefix) atomicAdd(&sh256[o & 0xffu], 1u);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t c = 0;
    for (int v = 255; v >= 0; --v) {
      if (c + sh256[v] >= need_tie) {
        s_low = uint32_t(v);
        s_above3 = c;
        break;
      }
      c += sh256[v];
    }
    s_gt_seen = 0;
    s_eq_seen = 0;
  }
  __syncthreads();
  const uint32_t ostar = (prefix << 8) | s_low;
  const uint32_t r_eq = need_tie - s_above3;  // entries equal to o* to keep
  for (int64_t base = 0; base < n; base += NT) {
    const int64_t i = base + threadIdx.x;
    const uint32_t o = i < n ? ord_f32(sc[i]) : 0u;
    const bool gt = i < n && o > ostar;
    const bool eq = i < n && o == ostar;
    uint32_t ngt, neq;
    const uint32_t gt_before = s_gt_seen + block_exclusive_scan<NT>(gt ? 1u : 0u, &ngt);
    const uint32_t eq_before = s_eq_seen + block_exclusive_scan<NT>(eq ? 1u : 0u, &neq);
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

// ------------------------------------------------------------------ paged, ragged scoring
// Sequence b of a ragged batch has n_b = max(0, floor((t_b - window) /
// stride)) keys, stored in pages of a pool: key i is pool row table[b][i /
// page] * page + i % page.  Only sequences with n_b > k need scores.  Their
// keys are laid end to end, each sequence padded to a multiple of 64 keys
// (the padding is masked), and the whole range is split evenly over one wave
// of CTAs, as in the dense-layout kernel: a CTA walks its range one sequence
// segment at a time with a shared-memory histogram flushed per segment.
// Segments start at multiples of 64 keys of their sequence and pages hold
// multiples of 64 rows, so a group of 16 keys never straddles two pages: each
// group resolves its page with one table load.  Keys of a page number outside
// the pool score -inf (and flag DSV4KV_DEV_BAD_PAGE).
constexpr int kMaxPagedBatch = 1024;
constexpr int kPagedAlign = 64;

__device__ __forceinline__ int64_t ragged_entries(const int64_t* t_seq, int b, int64_t t_max, int window, int stride,
                                                  int64_t n_max, uint32_t* status) {
  int64_t t = t_seq[b];
  if (t < 0 || t > t_max) {
    set_status(status, DSV4KV_DEV_BAD_LENGTH);
    t = t < 0 ? 0 : t_max;
  }
  return t > window ? min(n_max, (t - window) / stride) : 0;
}

struct PagedKeys {
  const void* codes;       // pool rows: bf16 [rows][128] or fp4 codes [rows][64]
  const uint8_t* scales;   // fp4: [rows][8]
  const int32_t* table;
  int page, tstride;
  int64_t pages;
};

// Pool row of key i of sequence b (-1: a page number outside the pool).  The
// page numbers of the segment being scored are staged in shared memory
// (pg_s[j] = the table entry of page pg0 + j) when they fit, else read from
// the table.
constexpr int kPageStage = 512;
__device__ __forceinline__ int64_t paged_key_row(const PagedKeys& pk, int b, int64_t i, const int32_t* pg_s,
                                                 int64_t pg0) {
  const int64_t pi = i / pk.page;
  const int32_t pg = pg_s ? pg_s[pi - pg0] : __ldg(pk.table + size_t(b) * pk.tstride + size_t(pi));
  if (pg < 0 || pg >= pk.pages) return -1;
  return int64_t(pg) * pk.page + i % pk.page;
}

// bf16 keys [i0, i0 + cnt) of sequence b (i0 a multiple of 64; keys >= n_b
// masked): the loop of score_segment_bf16 with a page lookup per group of 16.
template <int U>
__device__ __forceinline__ void score_segment_paged_bf16(const uint16_t* __restrict__ qrow, const PagedKeys& pk,
                                                         int b, int64_t i0, int64_t cnt, int64_t n_b, float* sc,
                                                         uint32_t* sh, uint64_t pol, uint32_t* status,
                                                         const int32_t* pg_s, int64_t pg0) {
  static_assert(U == 8, "two half-warps of 8 keys: a group of 16 keys");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int half = lane >> 4, l16 = lane & 15;
  const int my_key = (l16 >> 1) & 7;
  const bool writer = !(lane & 1);
  const uint16_t* keys = static_cast<const uint16_t*>(pk.codes) + 8 * l16;
  float q[8];
  {
    const uint4 v = *reinterpret_cast<const uint4*>(qrow + 8 * l16);
    q[0] = bf16lo(v.x); q[1] = bf16hi(v.x); q[2] = bf16lo(v.y); q[3] = bf16hi(v.y);
    q[4] = bf16lo(v.z); q[5] = bf16hi(v.z); q[6] = bf16lo(v.w); q[7] = bf16hi(v.w);
  }
  const int64_t valid = min(cnt, n_b - i0);  // keys of the segment that exist
  auto load = [&](int64_t j, uint4 (&v)[U], int64_t& row0) {
    // (a group of padding keys past the sequence's end looks up no page)
    row0 = 16 * j < valid ? paged_key_row(pk, b, i0 + 16 * j, pg_s, pg0) : 0;
    if (row0 < 0) set_status(status, DSV4KV_DEV_BAD_PAGE);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t key = 16 * j + U * half + u;
      v[u] = (row0 >= 0 && key < valid) ? ld_once_v4(keys + size_t(row0 + U * half + u) * 128, pol)
                                        : make_uint4(0, 0, 0, 0);
    }
  };
  auto process = [&](int64_t j, const uint4 (&v)[U], int64_t row0) {
    float p[U];
#pragma unroll
    for (int u = 0; u < U; ++u) p[u] = dot8_bf16(v[u], q);
    float s = reduce16_transposed<U>(p, l16) + 0.0f;  // -0 -> +0
    if (row0 < 0) s = -INFINITY;
    const int64_t key = 16 * j + U * half + my_key;
    if (writer && key < valid) {
      sc[key] = s;
      atomicAdd(&sh[ord_f32(s) >> 20], 1u);
    }
  };
  const int64_t ngroups = (cnt + 15) / 16;
  uint4 va[U], vb[U];
  int64_t ra = 0, rb = 0;
  int64_t j = warp;
  if (j < ngroups) load(j, va, ra);
  while (j < ngroups) {
    if (j + nwarps < ngroups) load(j + nwarps, vb, rb);
    process(j, va, ra);
    j += nwarps;
    if (j >= ngroups) break;
    if (j + nwarps < ngroups) load(j + nwarps, va, ra);
    process(j, vb, rb);
    j += nwarps;
  }
}

// fp4 keys: a quarter warp per key (lane l4 owns channels [32 l4, 32 l4 + 32)),
// 4 keys per quad and 32 per warp iteration (two iterations per group of 64
// are within one page).
__device__ __forceinline__ void score_segment_paged_fp4(const uint16_t* __restrict__ qrow, const PagedKeys& pk, int b,
                                                        int64_t i0, int64_t cnt, int64_t n_b, float* sc,
                                                        uint32_t* sh, uint64_t pol, uint32_t* status,
                                                        const int32_t* pg_s, int64_t pg0) {
  constexpr int U = 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int quad = lane >> 2, l4 = lane & 3;
  uint32_t qp[16];
  {
    const uint16_t* qb = qrow + 32 * l4;
#pragma unroll
    for (int j = 0; j < 16; ++j) qp[j] = f32x2_to_f16x2(bf16f(qb[2 * j]), bf16f(qb[2 * j + 1]));
  }
  const uint8_t* codes = static_cast<const uint8_t*>(pk.codes) + 16 * l4;
  const uint8_t* scales = pk.scales + 2 * l4;
  const int64_t valid = min(cnt, n_b - i0);
  auto load = [&](int64_t j, uint4 (&v)[U], uint32_t (&s2)[U], int64_t& row0) {
    // (a group of padding keys past the sequence's end looks up no page)
    row0 = 32 * j < valid ? paged_key_row(pk, b, i0 + 32 * j, pg_s, pg0) : 0;
    if (row0 < 0) set_status(status, DSV4KV_DEV_BAD_PAGE);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t key = 32 * j + 8 * u + quad;
      const bool ok = row0 >= 0 && key < valid;
      const size_t r = size_t(ok ? row0 + 8 * u + quad : 0);
      v[u] = ok ? ld_once_v4(codes + r * 64, pol) : make_uint4(0, 0, 0, 0);
      s2[u] = ok ? ld_once_u16(scales + r * 8, pol) : 0u;
    }
  };
  auto process = [&](int64_t j, const uint4 (&v)[U], const uint32_t (&s2)[U], int64_t row0) {
    float pr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t acc0 = 0, acc1 = 0;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        uint32_t h[4];
        e2m1x8_unpack(w[wi], h);
#pragma unroll
        for (int by = 0; by < 4; ++by) {
          if (wi < 2) acc0 = hfma2(qp[4 * wi + by], h[by], acc0);
          else acc1 = hfma2(qp[4 * wi + by], h[by], acc1);
        }
      }
      pr[u] = scaled_group_sums(acc0, acc1, s2[u]);
    }
    const bool bb1 = l4 & 2, bb0 = l4 & 1;
    float k2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) k2[i] = (bb1 ? pr[2 + i] : pr[i]) + __shfl_xor_sync(kFull, bb1 ? pr[i] : pr[2 + i], 2);
    float s = (bb0 ? k2[1] : k2[0]) + __shfl_xor_sync(kFull, bb0 ? k2[0] : k2[1], 1) + 0.0f;
    if (row0 < 0) s = -INFINITY;
    const int64_t key = 32 * j + 8 * l4 + quad;  // lane l4 ends with key u = l4
    if (key < valid) {
      sc[key] = s;
      atomicAdd(&sh[ord_f32(s) >> 20], 1u);
    }
  };
  const int64_t ngroups = (cnt + 31) / 32;
  uint4 va[U], vb[U];
  uint32_t sa[U], sb2[U];
  int64_t ra = 0, rb = 0;
  int64_t j = warp;
  if (j < ngroups) load(j, va, sa, ra);
  while (j < ngroups) {
    if (j + nwarps < ngroups) load(j + nwarps, vb, sb2, rb);
    process(j, va, sa, ra);
    j += nwarps;
    if (j >= ngroups) break;
    if (j + nwarps < ngroups) load(j + nwarps, va, sa, ra);
    process(j, vb, sb2, rb);
    j += nwarps;
  }
}

template <int FMT>
__global__ void __launch_bounds__(256) index_score_paged(const uint16_t* __restrict__ qidx, const PagedKeys pk,
                                                         const int64_t* __restrict__ t_seq, int64_t t_max, int window,
                                                         int stride, int64_t n_max, int k, int batch,
                                                         float* __restrict__ scores, uint32_t* __restrict__ hist,
                                                         uint32_t* __restrict__ status) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ int64_t s_pre[kMaxPagedBatch + 1];  // flattened start of every sequence; [batch] = the total
  __shared__ int32_t s_pg[kPageStage];           // the page numbers of the segment being scored
  pdl_trigger();
  pdl_wait();
  {
    constexpr int PER = kMaxPagedBatch / 256;
    int64_t c[PER], sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int b = PER * threadIdx.x + j;
      const int64_t n_b = b < batch ? ragged_entries(t_seq, b, t_max, window, stride, n_max, nullptr) : 0;
      c[j] = n_b > k ? (n_b + kPagedAlign - 1) / kPagedAlign * kPagedAlign : 0;
      sum += c[j];
    }
    // exclusive scan of the per-thread sums (in units of kPagedAlign keys, which fit 32 bits)
    uint32_t total;
    int64_t run = int64_t(block_exclusive_scan<256>(uint32_t(sum / kPagedAlign), &total)) * kPagedAlign;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int b = PER * threadIdx.x + j;
      if (b < batch) s_pre[b] = run;
      run += c[j];
    }
    if (threadIdx.x == 0) s_pre[batch] = int64_t(total) * kPagedAlign;
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const int64_t total = s_pre[batch];
  // the CTA's range: whole multiples of kPagedAlign keys
  const int64_t units = total / kPagedAlign;
  const int64_t per = (units + gridDim.x - 1) / gridDim.x * kPagedAlign;
  const int64_t g0 = min(total, int64_t(blockIdx.x) * per), g1 = min(total, g0 + per);
  const uint64_t pol = l2_evict_first_policy();  // keys are read once
  const size_t srow = size_t(score_stride(n_max));
  int b = 0;
  {  // the sequence holding g0: the last b with s_pre[b] <= g0
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= g0) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
  }
  int b_last = -1;
  for (int64_t s0 = g0; s0 < g1 && b < batch;) {
    const int64_t e = s_pre[b + 1];
    if (e <= s0) {  // an empty (or finished) sequence
      ++b;
      continue;
    }
    const int64_t s1 = min(g1, e);
    const int64_t i0 = s0 - s_pre[b];
    const int64_t n_b = ragged_entries(t_seq, b, t_max, window, stride, n_max, status);
    if (b_last >= 0) flush_histogram(sh, hist + size_t(b_last) * kHistBins);  // (starts with a block barrier)
    // stage the segment's page numbers (the keys that exist) in shared memory
    const int64_t pg0 = i0 / pk.page;
    const int64_t last = min(s1 - s0, n_b - i0);
    const int64_t npg = last > 0 ? (i0 + last - 1) / pk.page - pg0 + 1 : 0;
    const bool staged = npg <= kPageStage;
    if (staged)
      for (int64_t j = threadIdx.x; j < npg; j += blockDim.x)
        s_pg[j] = __ldg(pk.table + size_t(b) * pk.tstride + size_t(pg0 + j));
    __syncthreads();
    const int32_t* pg_s = staged ? s_pg : nullptr;
    if constexpr (FMT == DSV4KV_BF16)
      score_segment_paged_bf16<8>(qidx + size_t(b) * 128, pk, b, i0, s1 - s0, n_b, scores + size_t(b) * srow + i0, sh,
                                  pol, status, pg_s, pg0);
    else
      score_segment_paged_fp4(qidx + size_t(b) * 128, pk, b, i0, s1 - s0, n_b, scores + size_t(b) * srow + i0, sh, pol,
                              status, pg_s, pg0);
    __syncthreads();  // s_pg is rewritten for the next segment only after every warp used it
    b_last = b;
    s0 = s1;
  }
  if (b_last >= 0) flush_histogram(sh, hist + size_t(b_last) * kHistBins);
}

// (t_seq != null: a ragged batch, sequence b selects among its own n_b <=
// n_max entries; the score rows keep the stride of n_max.)
__global__ void __launch_bounds__(kSelThreads, 1) index_select(const float* __restrict__ scores, int64_t n_max, int k,
                                                            int64_t chunk, uint32_t* __restrict__ hist,
                                                            int32_t* __restrict__ idx_out,
                                                            int32_t* __restrict__ count_out,
                                                            uint32_t* __restrict__ status,
                                                            uint32_t* __restrict__ tail_ctr,
                                                            const int64_t* __restrict__ t_seq, int64_t t_max,
                                                            int window, int stride) {
  extern __shared__ __align__(16) uint64_t stage[];  // the tie list; kSelWarps lists of kWarpCap (the
                                                     // warps' runs); the leader's receive buffer
  __shared__ uint32_t s_wcnt[kSelWarps];
  __shared__ uint32_t s_rcnt[kMaxClusterSel];  // leader: the count each CTA pushed (~0u: overflow)
  __shared__ __align__(16) uint32_t sh[kHistBins];
  __shared__ uint32_t s_h3[256];  // leader: histogram of the low 8 code bits at the 24-bit prefix
  __shared__ uint32_t s_low, s_above3;
  __shared__ uint32_t s_pre[kMaxClusterSel + 1];

  const int b = blockIdx.y;
  const uint32_t rank = cluster_rank();
  const uint32_t csize = gridDim.x;  // one cluster spans the sequence's CTAs
  uint32_t* hb = hist + size_t(b) * kHistBins;
  const float* sc = scores + size_t(b) * size_t(score_stride(n_max));
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *tail_ctr = 0;  // the score kernel's queue, for the next call
  const int64_t n = t_seq ? ragged_entries(t_seq, b, t_max, window, stride, n_max, nullptr) : n_max;
  if (n <= k) {
    // a ragged sequence with no more entries than k: all of them (the score
    // kernel left its histogram untouched).  The whole cluster takes this
    // branch, before any cluster barrier.
    if (rank == 0) {
      int32_t* out = idx_out + size_t(b) * k;
      for (int i = threadIdx.x; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
      if (threadIdx.x == 0 && count_out) count_out[b] = int32_t(n);
    }
    return;
  }
  const uint32_t kk = uint32_t(k);
  const int64_t n0 = min(n, int64_t(rank) * chunk), n1 = min(n, n0 + chunk);
  cluster_arrive_relaxed();  // this CTA has started (waited for before the first remote store)

  // 1) every warp owns a contiguous run of the CTA's chunk; the first
  //    batches of its run are in flight while the histogram is read
  const int warp = threadIdx.x >> 5;
  const int64_t wspan = ((n1 - n0 + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
  const int64_t w0 = min(n1, n0 + int64_t(warp) * wspan), w1 = min(n1, w0 + wspan);
  const int64_t nbat = (w1 - w0 + kSelWarpSpan - 1) / kSelWarpSpan;
  float* ring = reinterpret_cast<float*>(stage) + size_t(warp) * kRing * kSelWarpSpan;
  HistLoad<kSelThreads> hl;
  hl.fetch(hb);  // first: the threshold waits for it, the batches are needed only after
#pragma unroll
  for (int t = 0; t < kRing - 1; ++t) {
    if (t < nbat) warp_issue_batch(sc, w0 + int64_t(t) * kSelWarpSpan, w1, ring + t * kSelWarpSpan);
    cp_async_commit();
  }
  hl.store(sh);
  __syncthreads();
  uint32_t above1;
  const int bin1 = find_threshold_bin<kSelThreads>(sh, kk, &above1);

  // 2) each warp filters its run into its own index-ordered list (no block
  //    barrier); the lists are then concatenated in warp order, which is
  //    index order
  uint64_t* wl = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage) + kRingBytes) + warp * kWarpCap;
  uint32_t wc = 0;
  for (int64_t t = 0; t < nbat; ++t) {
    if (t + kRing - 1 < nbat)
      warp_issue_batch(sc, w0 + (t + kRing - 1) * kSelWarpSpan, w1, ring + ((t + kRing - 1) % kRing) * kSelWarpSpan);
    cp_async_commit();
    cp_async_wait_group<kRing - 1>();  // batch t has landed (this lane's pieces)
    __syncwarp();                      // ... and every lane's
    uint32_t o[kSelBatch];
    warp_read_batch(ring + (t % kRing) * kSelWarpSpan, o);
    __syncwarp();  // the slot is read before it is refilled
    wc = warp_stage_batch(o, w0 + t * kSelWarpSpan, w1, bin1, wc, wl);
  }
  cp_async_wait_group<0>();  // nothing left in flight (batches past the run were never issued)
  if (lane == 0) s_wcnt[warp] = wc;
  __syncthreads();
  // 3) every CTA pushes its warps' lists, concatenated in warp order, into
  //    its region of the leader's receive buffer (remote shared-memory stores),
  //    and its count; a list or region that overflowed sends the sequence to
  //    the exact fallback
  const uint32_t regcap = uint32_t(kRecvCap) / csize;
  uint64_t* recv = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage) + kRingBytes) + kSelStage;
  {
    uint32_t off = 0, tot = 0;
    bool over = false;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
      const uint32_t c = s_wcnt[w];
      off += w < warp ? c : 0u;
      tot += c;
      over |= c > uint32_t(kWarpCap);
    }
    over |= tot > regcap;
    const uint32_t mine = min(wc, uint32_t(kWarpCap));
    const uint32_t dst = dsmem_addr(recv + size_t(rank) * regcap, 0);
    cluster_wait();  // every CTA of the cluster (the leader among them) has started
    if (!over)
      for (uint32_t i = lane; i < mine; i += 32) st_dsmem_u64(dst + 8u * (off + i), wl[i]);
    if (threadIdx.x == 0) st_dsmem_u32(dsmem_addr(&s_rcnt[rank], 0), over ? 0xffffffffu : tot);
  }
  if (rank == 0) {  // the leader's resolve state, cleared while the other CTAs finish
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) sh[i] = 0;
    for (int i = threadIdx.x; i < 256; i += kSelThreads) s_h3[i] = 0;
  }
  cluster_sync();  // every list is in the leader's shared memory
  if (rank != 0) {
    // leave the histogram zeroed for the next call (every CTA read it before the barrier)
    if (rank == 1)
      for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) hb[i] = 0;
    return;
  }

  // 4) the leader reads the regions in rank order (= index order)
  uint64_t c[kResPer];
  uint32_t total = 0;
  bool fits = true;
  if (threadIdx.x < 32) {  // one warp scan of the counts gives the offsets
    const uint32_t cnt = threadIdx.x < csize ? s_rcnt[threadIdx.x] : 0u;
    const bool bad = __any_sync(kFull, cnt == 0xffffffffu);
    const uint32_t incl = warp_inclusive_scan(bad ? 0u : cnt);
    if (threadIdx.x < csize) s_pre[threadIdx.x] = incl - (bad ? 0u : cnt);
    if (threadIdx.x == csize - 1) s_pre[csize] = bad ? 0xffffffffu : incl;
  }
  __syncthreads();
  total = s_pre[csize];
  fits = total <= uint32_t(kCandCap);
  const int J = int((total + kSelThreads - 1) / kSelThreads);  // candidate rounds in use (block-uniform)
  if (fits) {
    // the region of every position (offsets in registers, a branch-free
    // search: offsets are non-decreasing, the last one <= g holds g)
    uint32_t pre[kMaxClusterSel];
#pragma unroll
    for (int i = 0; i < kMaxClusterSel; ++i) pre[i] = i < int(csize) ? s_pre[i] : 0xffffffffu;
#pragma unroll
    for (int j = 0; j < kResPer; ++j) {
      c[j] = 0ull;
      if (j >= J) continue;
      const uint32_t g = threadIdx.x + uint32_t(j) * kSelThreads;
      uint32_t r = 0, base = 0;
#pragma unroll
      for (int i = 1; i < kMaxClusterSel; ++i) {
        const bool past = pre[i] <= g;
        r = past ? uint32_t(i) : r;
        base = past ? pre[i] : base;
      }
      if (g < total) c[j] = recv[size_t(r) * regcap + (g - base)];
    }
  }

  // 5) resolve: the exact threshold code T from two more histogram levels
  //    over the candidates; codes above T are kept, and of the codes equal to
  //    T (equal scores) the first need_eq by position (= by index)
  int32_t* out = idx_out + size_t(b) * k;
  const uint32_t need1 = kk - above1;  // still needed from bin1 (>= 1)
  const uint32_t lt = (1u << lane) - 1u;
  bool ok = false;
  uint32_t prefix = 0, need_tie = 0;
  if (fits) {
    // bits 8-19 of the codes in bin1 (every entry of bin1 is a candidate)
#pragma unroll
    for (int j = 0; j < kResPer; ++j) {
      const uint32_t g = threadIdx.x + uint32_t(j) * kSelThreads;
      const uint32_t o = uint32_t(c[j] >> 32);
      if (j < J) hist_add_warp(sh, g < total && int(o >> 20) == bin1, (o >> 8) & 0xfffu);
    }
    __syncthreads();
    uint32_t above2;
    const int bin2 = find_threshold_bin<kSelThreads>(sh, need1, &above2);
    prefix = (uint32_t(bin1) << 12) | uint32_t(bin2);  // 24-bit threshold prefix
    need_tie = need1 - above2;                          // >= 1
    // bits 0-7 of the codes at the prefix
#pragma unroll
    for (int j = 0; j < kResPer; ++j) {
      const uint32_t g = threadIdx.x + uint32_t(j) * kSelThreads;
      const uint32_t o = uint32_t(c[j] >> 32);
      if (j < J) hist_add_warp(s_h3, g < total && (o >> 8) == prefix, o & 0xffu);
    }
    __syncthreads();
    if (warp == 0) {  // lane l owns bins 255 - 8l - 7 .. 255 - 8l (descending lane order)
      uint32_t v[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = s_h3[255 - 8 * lane - i];
        sum += v[i];
      }
      const uint32_t incl = warp_inclusive_scan(sum);
      uint32_t cnt = incl - sum;
      if (cnt < need_tie && incl >= need_tie) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cnt < need_tie && cnt + v[i] >= need_tie) {
            s_low = uint32_t(255 - 8 * lane - i);
            s_above3 = cnt;
          }
          cnt += v[i];
        }
      }
    }
    __syncthreads();
    const uint32_t tcode = (prefix << 8) | s_low;
    const uint32_t need_eq = need_tie - s_above3;  // codes equal to T to keep (>= 1)
    // one ordered scan counts, before every position, the codes above T and
    // the codes equal to T; an entry's output slot is (above before) +
    // min(equal before, need_eq), so the kept entries come out in index order
    uint32_t mg[kResPer], me[kResPer], off[kResPer];
#pragma unroll
    for (int j = 0; j < kResPer; ++j) {
      const uint32_t g = threadIdx.x + uint32_t(j) * kSelThreads;
      const uint32_t o = uint32_t(c[j] >> 32);
      mg[j] = j < J ? __ballot_sync(kFull, g < total && o > tcode) : 0u;
      me[j] = j < J ? __ballot_sync(kFull, g < total && o == tcode) : 0u;
    }
    const uint32_t tot = ordered_offsets_pair<kSelThreads, kResPer>(mg, me, off);
    const uint32_t got = (tot >> 16) + min(tot & 0xffffu, need_eq);
#pragma unroll
    for (int j = 0; j < kResPer; ++j) {
      const uint32_t gt_before = (off[j] >> 16) + __popc(mg[j] & lt);
      const uint32_t eq_before = (off[j] & 0xffffu) + __popc(me[j] & lt);
      const bool gt = (mg[j] >> lane) & 1u, eq = (me[j] >> lane) & 1u;
      if (gt || (eq && eq_before < need_eq)) {
        const uint32_t at = gt_before + min(eq_before, need_eq);
        if (at < kk) out[at] = int32_t(0xffffffffu - uint32_t(c[j]));
      }
    }
    if (threadIdx.x == 0 && got != kk) set_status(status, DSV4KV_DEV_INCONSISTENT);
    ok = true;
  }
  __syncthreads();
  if (!ok) {
    if (!fits) {
      // the candidates did not fit: the second-level threshold from all scores
      for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) sh[i] = 0;
      __syncthreads();
      for (int64_t i = threadIdx.x; i < n; i += kSelThreads) {
        const uint32_t o = ord_f32(sc[i]);
        if (int(o >> 20) == bin1) atomicAdd(&sh[(o >> 8) & 0xfffu], 1u);
      }
      __syncthreads();
      uint32_t above2;
      const int bin2 = find_threshold_bin<kSelThreads>(sh, need1, &above2);
      prefix = (uint32_t(bin1) << 12) | uint32_t(bin2);
      need_tie = need1 - above2;
    }
    select_by_scan<kSelThreads>(sc, n, prefix, need_tie, kk, out, sh, status);
  }
  for (int i = int(kk) + threadIdx.x; i < k; i += kSelThreads) out[i] = -1;
  if (threadIdx.x == 0 && count_out) count_out[b] = int32_t(kk);
  // 6) leave the histogram zeroed for the next call (a one-CTA cluster has no helper)
  if (csize == 1)
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) hb[i] = 0;
}

__global__ void index_fill_all(int64_t n_max, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ count_out,
                               const int64_t* __restrict__ t_seq, int64_t t_max, int window, int stride,
                               uint32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.y;
  const int64_t n = t_seq ? ragged_entries(t_seq, b, t_max, window, stride, n_max, status) : n_max;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < k; i += gridDim.x * blockDim.x)
    idx_out[size_t(b) * k + i] = i < n ? i : -1;
  if (count_out && blockIdx.x == 0 && threadIdx.x == 0) count_out[b] = int32_t(n);
}

// ------------------------------------------------------------------ pool re-index
// [P3] CSA2: a "Reindex" layer keeps its indexing inside the candidate pool
// built by the first layer in Full mode (the layers share the indexer keys).
// One thread-block cluster of C <= 4 CTAs (512 threads) per sequence: CTA r
// gathers and scores the r-th part of the pool (ascending entry indices,
// negative = no entry; half a warp per bf16 key, a quarter warp per fp4 key)
// and pushes the order-preserving codes, its 12-bit histogram and its count
// into the leader's shared memory; after one cluster barrier the leader runs
// the exact selection: the 12-bit histogram gives the threshold bin, a second 12-bit
// histogram of that bin the 24-bit prefix, a 256-bin histogram of the
// entries at the prefix the threshold code, and the entries equal to it are
// taken in pool order (= entry order, so ties go to the lower entry); an
// ordered compaction over pool positions writes the result ascending.
constexpr int kPoolMax = 8192;
constexpr int kPoolPer = kPoolMax / kSelThreads;  // pool positions per thread
constexpr int kMaxPoolCluster = 4;
// dynamic shared memory: codes and entries of the pool, the CTAs' histograms (leader)
constexpr size_t kPoolDyn = (2 * size_t(kPoolMax) + size_t(kMaxPoolCluster) * kHistBins) * sizeof(uint32_t);

// The bin where the descending cumulative count of a 256-bin histogram first
// reaches `need`; *above = count in higher bins.  Warp 0 scans (8 bins per
// lane), one block barrier publishes the result.
__device__ int find_threshold_bin256(const uint32_t* h, uint32_t need, uint32_t* above) {
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int lo = 256 - 8 * (lane + 1);  // lane 0 owns the highest 8 bins
    uint32_t v[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = h[lo + i];
      sum += v[i];
    }
    const uint32_t incl = warp_inclusive_scan(sum);
    const uint32_t ex = incl - sum;
    if (ex < need && ex + sum >= need) {
      uint32_t c = ex;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (c < need && c + v[i] >= need) {
          s_bin = lo + i;
          s_above = c;
        }
        c += v[i];
      }
    }
  }
  __syncthreads();
  *above = s_above;
  const int r = s_bin;
  __syncthreads();
  return r;
}

// PER: pool positions per thread (PER x 512 >= the pool's capacity).  The
// kernel is latency-bound and its loops over the positions are unrolled, so
// pools of up to 2048 entries take PER = 4 (a quarter of the code of PER = 16).
template <int FMT, int PER>
__global__ void __launch_bounds__(kSelThreads, 1)
    index_pool_select(const uint16_t* __restrict__ qidx, const void* __restrict__ codes,
                      const uint8_t* __restrict__ kscales, int64_t key_rows, int64_t n,
                      const int32_t* __restrict__ pool, int pool_cap, int k, int32_t* __restrict__ idx_out,
                      int32_t* __restrict__ count_out, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint32_t psm[];
  uint32_t* pcode = psm;              // leader: kPoolMax order-preserving codes (0 = no entry)
  int32_t* pent = reinterpret_cast<int32_t*>(psm + kPoolMax);  // the pool's entries (this CTA's part; leader: all)
  uint32_t* hparts = psm + 2 * kPoolMax;                       // leader: the CTAs' histograms
  __shared__ __align__(16) uint32_t sh[kHistBins];
  __shared__ uint32_t s_cnt;
  __shared__ uint32_t s_cparts[kMaxPoolCluster];
  const int b = blockIdx.y;
  const uint32_t rank = cluster_rank(), csize = gridDim.x;  // one cluster spans the sequence's CTAs
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t* pb = pool + size_t(b) * pool_cap;
  // this CTA's part of the pool: [c0, c1), whole multiples of 32 positions
  const int part = ((pool_cap + int(csize) - 1) / int(csize) + 31) / 32 * 32;
  const int c0 = min(pool_cap, int(rank) * part), c1 = min(pool_cap, c0 + part);
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) sh[i] = 0;
  if (threadIdx.x == 0) s_cnt = 0;
  pdl_trigger();
  pdl_wait();
  cluster_arrive_relaxed();  // this CTA has started (waited for before the first remote store)
  // the pool (the leader reads all of it for the output and checks it: entries
  // in [0, n), ascending); the other CTAs read their part
  const int e0 = rank == 0 ? 0 : c0, e1 = rank == 0 ? pool_cap : c1;
  for (int j = e0 + int(threadIdx.x); j < e1; j += kSelThreads) {
    const int32_t e = pb[j];
    pent[j] = e;
    if (rank == 0) {
      if (e >= n) set_status(status, DSV4KV_DEV_BAD_INDEX);
      if (e >= 0 && j > 0 && !(pb[j - 1] >= 0 && pb[j - 1] < e)) set_status(status, DSV4KV_DEV_BAD_POOL);
    }
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster (the leader among them) has started
  const uint64_t pol = l2_evict_first_policy();
  if constexpr (FMT == DSV4KV_BF16) {
    // half-warp hw scores positions hw, hw + 32, ...; 16 keys in flight per
    // half-warp.  The loop bound is the same for every thread (positions past
    // the pool are masked) so that the shuffles always see the whole warp.
    constexpr int U = 16;
    const int half = lane >> 4, l16 = lane & 15, hw = 2 * warp + half;
    float q[8];
    {
      const uint4 v = *reinterpret_cast<const uint4*>(qidx + size_t(b) * 128 + 8 * l16);
      q[0] = bf16lo(v.x); q[1] = bf16hi(v.x); q[2] = bf16lo(v.y); q[3] = bf16hi(v.y);
      q[4] = bf16lo(v.z); q[5] = bf16hi(v.z); q[6] = bf16lo(v.w); q[7] = bf16hi(v.w);
    }
    const uint16_t* kb = static_cast<const uint16_t*>(codes) + size_t(b) * size_t(key_rows) * 128 + 8 * l16;
    for (int it = 0; it * 32 * U < c1 - c0; ++it) {
      const int j0 = c0 + hw + 32 * U * it;
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 32 * u;
        const int32_t e = j < c1 ? pent[j] : -1;
        v[u] = (e >= 0 && e < n) ? ld_once_v4(kb + size_t(e) * 128, pol) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 32 * u;
        float sc = dot8_bf16(v[u], q);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sc += __shfl_xor_sync(kFull, sc, o);
        sc += 0.0f;  // -0 -> +0
        if (l16 == 0 && j < c1) {
          const int32_t e = pent[j];
          const bool ok = e >= 0 && e < n;
          const uint32_t c = ok ? ord_f32(sc) : 0u;
          st_dsmem_u32(dsmem_addr(&pcode[j], 0), c);
          if (ok) {
            atomicAdd(&sh[c >> 20], 1u);
            atomicAdd(&s_cnt, 1u);
          }
        }
      }
    }
  } else {
    // fp4 keys: a quarter warp per key, lane l4 owns channels [32 l4, 32 l4 + 32);
    // a loop bound common to all threads, as above
    constexpr int U = 8;
    const int quad = threadIdx.x >> 2, l4 = lane & 3;  // 128 quads
    uint32_t qp[16];
    {
      const uint16_t* qb = qidx + size_t(b) * 128 + 32 * l4;
#pragma unroll
      for (int j = 0; j < 16; ++j) qp[j] = f32x2_to_f16x2(bf16f(qb[2 * j]), bf16f(qb[2 * j + 1]));
    }
    const uint8_t* cb = static_cast<const uint8_t*>(codes) + size_t(b) * size_t(key_rows) * 64 + 16 * l4;
    const uint8_t* sb = kscales + size_t(b) * size_t(key_rows) * 8 + 2 * l4;
    for (int it = 0; it * 128 * U < c1 - c0; ++it) {
      const int j0 = c0 + quad + 128 * U * it;
      uint4 v[U];
      uint32_t s2[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 128 * u;
        const int32_t e = j < c1 ? pent[j] : -1;
        const bool ok = e >= 0 && e < n;
        v[u] = ok ? ld_once_v4(cb + size_t(e) * 64, pol) : make_uint4(0, 0, 0, 0);
        s2[u] = ok ? ld_once_u16(sb + size_t(e) * 8, pol) : 0u;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 128 * u;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t acc0 = 0, acc1 = 0;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint32_t h[4];
          e2m1x8_unpack(w[wi], h);
#pragma unroll
          for (int by = 0; by < 4; ++by) {
            if (wi < 2) acc0 = hfma2(qp[4 * wi + by], h[by], acc0);
            else acc1 = hfma2(qp[4 * wi + by], h[by], acc1);
          }
        }
        float sc = scaled_group_sums(acc0, acc1, s2[u]);
        sc += __shfl_xor_sync(kFull, sc, 1);
        sc += __shfl_xor_sync(kFull, sc, 2);
        sc += 0.0f;
        if (l4 == 0 && j < c1) {
          const int32_t e = pent[j];
          const bool ok = e >= 0 && e < n;
          const uint32_t c = ok ? ord_f32(sc) : 0u;
          st_dsmem_u32(dsmem_addr(&pcode[j], 0), c);
          if (ok) {
            atomicAdd(&sh[c >> 20], 1u);
            atomicAdd(&s_cnt, 1u);
          }
        }
      }
    }
  }
  __syncthreads();
  // this CTA's histogram and count into the leader; one cluster barrier
  {
    const uint32_t hdst = dsmem_addr(hparts + size_t(rank) * kHistBins, 0);
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) st_dsmem_u32(hdst + 4u * uint32_t(i), sh[i]);
    if (threadIdx.x == 0) st_dsmem_u32(dsmem_addr(&s_cparts[rank], 0), s_cnt);
  }
  cluster_sync();  // every code, histogram and count is in the leader's shared memory
  if (rank != 0) return;
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) {
    uint32_t sum = 0;
    for (uint32_t r = 0; r < csize; ++r) sum += hparts[size_t(r) * kHistBins + i];
    sh[i] = sum;
  }
  if (threadIdx.x == 0) {
    uint32_t tot = 0;
    for (uint32_t r = 0; r < csize; ++r) tot += s_cparts[r];
    s_cnt = tot;
  }
  __syncthreads();
  const uint32_t cnt = s_cnt;
  const uint32_t kk = min(uint32_t(k), cnt);
  uint32_t c[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int pos = threadIdx.x + j * kSelThreads;
    c[j] = pos < pool_cap ? pcode[pos] : 0u;
  }
  // the threshold code o* and how many entries equal to it are needed
  uint32_t ostar = 1u, need_eq = 0xffffffffu;  // every valid entry (codes >= 1) when cnt <= k
  if (cnt > uint32_t(k)) {
    uint32_t above1, above2, above3;
    const int bin1 = find_threshold_bin<kSelThreads>(sh, kk, &above1);
    for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) sh[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (c[j] != 0u && int(c[j] >> 20) == bin1) atomicAdd(&sh[(c[j] >> 8) & 0xfffu], 1u);
    __syncthreads();
    const int bin2 = find_threshold_bin<kSelThreads>(sh, kk - above1, &above2);
    const uint32_t prefix = (uint32_t(bin1) << 12) | uint32_t(bin2);
    for (int i = threadIdx.x; i < 256; i += kSelThreads) sh[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (c[j] != 0u && (c[j] >> 8) == prefix) atomicAdd(&sh[c[j] & 0xffu], 1u);
    __syncthreads();
    const int bin3 = find_threshold_bin256(sh, kk - above1 - above2, &above3);
    ostar = (prefix << 8) | uint32_t(bin3);
    need_eq = kk - above1 - above2 - above3;
  }
  // ranks of the entries equal to o*, in pool order
  uint32_t m[PER], off[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) m[j] = __ballot_sync(kFull, cnt > uint32_t(k) && c[j] == ostar);
  ordered_offsets<kSelThreads, PER>(m, off);
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const bool eq = (m[j] >> lane) & 1u;
    const bool keep = cnt > uint32_t(k) ? (c[j] > ostar || (eq && off[j] + __popc(m[j] & lt) < need_eq)) : c[j] != 0u;
    m[j] = __ballot_sync(kFull, keep);
  }
  const uint32_t got = ordered_offsets<kSelThreads, PER>(m, off);
  int32_t* out = idx_out + size_t(b) * k;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if ((m[j] >> lane) & 1u) {
      const uint32_t at = off[j] + __popc(m[j] & lt);
      if (at < kk) out[at] = pent[threadIdx.x + j * kSelThreads];
    }
  }
  for (int i = int(kk) + threadIdx.x; i < k; i += kSelThreads) out[i] = -1;
  if (threadIdx.x == 0) {
    if (count_out) count_out[b] = int32_t(kk);
    if (got != kk) set_status(status, DSV4KV_DEV_INCONSISTENT);
  }
}

dsv4kv_status index_topk_pool_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n,
                                     const int32_t* pool, int pool_cap, int k, int32_t* idx_out, int32_t* count_out,
                                     void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (ws_bytes < 16) return set_error(DSV4KV_ERR_WORKSPACE, "index_topk_pool: workspace too small");
  if (pool_cap > kPoolMax)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_pool: pool of %d entries > %d", pool_cap, kPoolMax);
  uint32_t* status = static_cast<uint32_t*>(ws);
  static std::atomic<uint64_t> attr{0};  // one bit per device
  if (!done_on_device(attr)) {
    if (cudaFuncSetAttribute(index_pool_select<DSV4KV_BF16, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kPoolDyn)) != cudaSuccess ||
        cudaFuncSetAttribute(index_pool_select<DSV4KV_BF16, kPoolPer>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kPoolDyn)) != cudaSuccess ||
        cudaFuncSetAttribute(index_pool_select<DSV4KV_FP4_E2M1_G16, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kPoolDyn)) != cudaSuccess ||
        cudaFuncSetAttribute(index_pool_select<DSV4KV_FP4_E2M1_G16, kPoolPer>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPoolDyn)) != cudaSuccess)
      return check_launch("index_topk_pool: cudaFuncSetAttribute");
    mark_done_on_device(attr);
  }
  // C CTAs per sequence, as many as keep the grid within one CTA per SM
  const int csize = std::max(1, std::min(kMaxPoolCluster, sm_count() / std::max(batch, 1)));
  const dim3 grid{static_cast<unsigned>(csize), static_cast<unsigned>(batch)};
  const bool small = pool_cap <= 4 * kSelThreads;
  const void* kc = keys.codes;
  const uint8_t* ks = static_cast<const uint8_t*>(keys.scales);
  if (keys.fmt == DSV4KV_BF16) {
    if (small)
      launch_pdl_cluster(index_pool_select<DSV4KV_BF16, 4>, grid, dim3(kSelThreads), kPoolDyn, unsigned(csize), stream,
                         qidx, kc, ks, keys.rows, n, pool, pool_cap, k, idx_out, count_out, status);
    else
      launch_pdl_cluster(index_pool_select<DSV4KV_BF16, kPoolPer>, grid, dim3(kSelThreads), kPoolDyn, unsigned(csize),
                         stream, qidx, kc, ks, keys.rows, n, pool, pool_cap, k, idx_out, count_out, status);
  } else {
    if (small)
      launch_pdl_cluster(index_pool_select<DSV4KV_FP4_E2M1_G16, 4>, grid, dim3(kSelThreads), kPoolDyn, unsigned(csize),
                         stream, qidx, kc, ks, keys.rows, n, pool, pool_cap, k, idx_out, count_out, status);
    else
      launch_pdl_cluster(index_pool_select<DSV4KV_FP4_E2M1_G16, kPoolPer>, grid, dim3(kSelThreads), kPoolDyn,
                         unsigned(csize), stream, qidx, kc, ks, keys.rows, n, pool, pool_cap, k, idx_out, count_out,
                         status);
  }
  return check_launch("index_pool_select");
}

// ------------------------------------------------------------------ host side
struct IndexWs {
  uint32_t* status;
  uint32_t* hist;
  uint32_t* tail_ctr;  // claim counter of the bf16 score kernel's tail queue
  float* scores;
  size_t scores_off;   // byte offset of the scores: everything before must be zero between calls
  size_t bytes;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static IndexWs index_ws_layout(char* base, int batch, int64_t n, int k) {
  (void)k;
  IndexWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  };
  w.status = reinterpret_cast<uint32_t*>(take(16));
  w.hist = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * kHistBins * size_t(batch)));
  w.tail_ctr = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t)));
  w.scores_off = off;
  w.scores = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * size_t(score_stride(n))));
  w.bytes = off;
  return w;
}

size_t index_topk_ws_bytes(int batch, int64_t n, int k) { return index_ws_layout(nullptr, batch, n, k).bytes; }

// Bytes at the start of the workspace that must be zero before a call (status
// word, counters, histograms): everything before the scores.
size_t index_topk_zero_prefix_bytes(int batch) { return index_ws_layout(nullptr, batch, 1, 1).scores_off; }

static dsv4kv_status index_fill_launch(int batch, int64_t n, int k, int32_t* idx_out, int32_t* count_out,
                                       cudaStream_t stream, const Ragged& rg, uint32_t* status) {
  const dim3 grid((unsigned)((k + 255) / 256), (unsigned)batch);
  launch_pdl(index_fill_all, grid, dim3(256), 0, stream, n, k, idx_out, count_out, rg.t_seq, rg.t_max, rg.window,
             rg.stride, status);
  return check_launch("index_fill_all");
}

dsv4kv_status index_score_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n, int k,
                                 void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (n <= k) return DSV4KV_OK;  // every entry is selected: nothing to score
  const IndexWs w = index_ws_layout(static_cast<char*>(ws), batch, n, k);
  if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "index_score: workspace too small");
  const int sms = sm_count();
  // one CTA per SM streaming the keys through shared memory; the last
  // kTailPct % of every sequence (whole units of a stage's keys) goes to the
  // shared queue, whose histogram counts go straight to global memory: with
  // few sequences they would pile onto the few bins that hold most scores of
  // one histogram, so small batches use the even split alone
  if ((reinterpret_cast<uintptr_t>(qidx) | reinterpret_cast<uintptr_t>(keys.codes) |
       reinterpret_cast<uintptr_t>(keys.scales)) & 15)
    return set_error(DSV4KV_ERR_INVALID_ARG, "index_score: queries, codes and scales must be 16-byte aligned");
  auto launch = [&](auto traits, void (*kern)(const uint16_t*, const uint8_t*, const uint8_t*, int64_t, int64_t,
                                              int64_t, int, int64_t, float*, uint32_t*, uint32_t*, uint32_t*),
                    std::atomic<uint64_t>& attr_set) -> dsv4kv_status {
    using F = decltype(traits);
    if (!done_on_device(attr_set)) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(stream_smem<F>())) !=
          cudaSuccess)
        return check_launch("index_score: cudaFuncSetAttribute");
      mark_done_on_device(attr_set);
    }
    const int64_t n_tail = batch >= kTailMinBatch ? std::min<int64_t>(n, (n * kTailPct / 100) / F::kKeys * F::kKeys) : 0;
    const int64_t n_h = n - n_tail;
    const int64_t total = int64_t(batch) * n_h;
    const int64_t per_cta = std::max<int64_t>(F::kKeys, (total + sms - 1) / sms);
    launch_pdl(kern, dim3(unsigned(sms)), dim3(StreamLayout<F>::kThreads), stream_smem<F>(), stream, qidx,
               static_cast<const uint8_t*>(keys.codes), static_cast<const uint8_t*>(keys.scales), keys.rows, n, n_h,
               batch, per_cta, w.scores, w.hist, w.tail_ctr, w.status);
    return DSV4KV_OK;
  };
  static std::atomic<uint64_t> attr_bf16{0}, attr_fp4{0};
  const dsv4kv_status st = keys.fmt == DSV4KV_BF16
                               ? launch(StreamBf16{}, index_score_stream<StreamBf16>, attr_bf16)
                               : launch(StreamFp4{}, index_score_stream<StreamFp4>, attr_fp4);
  if (st != DSV4KV_OK) return st;
  return check_launch("index_score");
}

dsv4kv_status index_select_launch(int batch, int64_t n, int k, int32_t* idx_out, int32_t* count_out, void* ws,
                                  size_t ws_bytes, cudaStream_t stream, const Ragged& rg) {
  if (n <= k)
    return index_fill_launch(batch, n, k, idx_out, count_out, stream, rg,
                             ws_bytes >= 16 ? static_cast<uint32_t*>(ws) : nullptr);
  const IndexWs w = index_ws_layout(static_cast<char*>(ws), batch, n, k);
  if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "index_select: workspace too small");
  const int sms = sm_count();
  // selection: one cluster of C CTAs per sequence, chunks of whole 4096-score batches
  static std::atomic<int> max_cluster_dev[64];  // per device; 0 = not set up yet
  std::atomic<int>& max_cluster_slot = max_cluster_dev[current_device()];
  int max_cluster = max_cluster_slot.load(std::memory_order_acquire);
  if (max_cluster == 0) {
    if (cudaFuncSetAttribute(index_select, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSelDyn)) != cudaSuccess)
      return check_launch("index_select: cudaFuncSetAttribute");
    max_cluster = 8;
    if (cudaFuncSetAttribute(index_select, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(kMaxClusterSel, 1);
      cfg.blockDim = dim3(kSelThreads);
      cfg.dynamicSmemBytes = kSelDyn;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kMaxClusterSel;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, index_select, &cfg) == cudaSuccess && clusters > 0)
        max_cluster = kMaxClusterSel;
    }
    cudaGetLastError();  // a refused query only means the portable size
    max_cluster_slot.store(max_cluster, std::memory_order_release);
  }
  // at most one CTA per SM in all (the leader's registers allow one per SM)
  const int64_t per_seq = std::max<int64_t>(1, std::min<int64_t>(max_cluster, sms / std::max(batch, 1)));
  const int64_t units_per_cta = std::max<int64_t>(1, (n + per_seq * kSelChunkUnit - 1) / (per_seq * kSelChunkUnit));
  const int64_t chunk = units_per_cta * kSelChunkUnit;
  const unsigned ctas = unsigned((n + chunk - 1) / chunk);
  launch_pdl_cluster(index_select, dim3(ctas, unsigned(batch)), dim3(kSelThreads), kSelDyn, ctas, stream,
                     (const float*)w.scores, n, k, chunk, w.hist, idx_out, count_out, w.status, w.tail_ctr, rg.t_seq,
                     rg.t_max, rg.window, rg.stride);
  return check_launch("index_select");
}


dsv4kv_status index_topk_launch(const uint16_t* qidx, const dsv4kv_cache& keys, int batch, int64_t n, int k,
                                int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  const dsv4kv_status st = index_score_launch(qidx, keys, batch, n, k, ws, ws_bytes, stream);
  if (st != DSV4KV_OK) return st;
  return index_select_launch(batch, n, k, idx_out, count_out, ws, ws_bytes, stream, Ragged{});
}

dsv4kv_status index_topk_paged_launch(const uint16_t* qidx, const dsv4kv_cache& pool, const PageDesc& pg, int batch,
                                      const Ragged& rg, int k, int32_t* idx_out, int32_t* count_out, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
  const int64_t n_max = rg.t_max > rg.window ? (rg.t_max - rg.window) / rg.stride : 0;
  if (batch > kMaxPagedBatch)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "index_topk_paged: batch %d > %d", batch, kMaxPagedBatch);
  if (n_max > k) {
    const IndexWs w = index_ws_layout(static_cast<char*>(ws), batch, n_max, k);
    if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "index_topk_paged: workspace too small");
    const PagedKeys pk{pool.codes, static_cast<const uint8_t*>(pool.scales), pg.table, pg.page_rows, pg.table_stride,
                       pg.pool_pages};
    // one wave of persistent CTAs draining the unit queue
    auto kern = pool.fmt == DSV4KV_BF16 ? index_score_paged<DSV4KV_BF16> : index_score_paged<DSV4KV_FP4_E2M1_G16>;
    static std::atomic<int> occ_dev[2][64];  // per format and device; 0 = not queried yet
    std::atomic<int>& slot = occ_dev[pool.fmt == DSV4KV_BF16 ? 0 : 1][current_device()];
    int occ = slot.load(std::memory_order_relaxed);
    if (occ == 0) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, 0) != cudaSuccess || occ < 1) occ = 1;
      slot.store(occ, std::memory_order_relaxed);
    }
    launch_pdl(kern, dim3(unsigned(sm_count() * occ)), dim3(256), 0, stream, qidx, pk, rg.t_seq, rg.t_max, rg.window,
               rg.stride, n_max, k, batch, w.scores, w.hist, w.status);
    const dsv4kv_status st = check_launch("index_score_paged");
    if (st != DSV4KV_OK) return st;
  }
  return index_select_launch(batch, n_max, k, idx_out, count_out, ws, ws_bytes, stream, rg);
}

}  // namespace dsv4kv
