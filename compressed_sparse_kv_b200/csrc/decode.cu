// Shared-K/V decode attention over compressed entries plus the window.
//
// [P2] Step 3: one cached vector S_j serves as the key (score = Q . S_j) and
// as the value; [P1] "The sliding window": every layer also reads 128 exact
// recent rows; [P1] "Shared key and value": an inverse RoPE is applied to the
// output; [P1] "c4a" / "c128a" and [P2] Step 5: c4a reads the top-k selected
// entries, c128a reads all of them.
//
// One CTA per (sequence, split) runs over a contiguous range of 64-row tiles
// of that sequence's row list (selected or all compressed rows, then window
// rows).  Per tile:
//   * warp 0 gathers the 64 rows into shared memory with TMA tile::gather4
//     (4 rows x 64 channels per copy, 128-byte swizzle);
//   * warp 1 (one thread) issues tcgen05.mma: S = Q . R^T (M = 64 heads,
//     N = 64 rows, K = 512) into TMEM, then O^T += R^T . P^T (M = 128 channels
//     x 4 tiles, N = 64 heads, K = 64 rows) — the SAME shared-memory tile is
//     the K-major B operand of the first product and the MN-major A operand
//     of the second, which is the shared-K/V saving;
//   * warps 2-5 run the online softmax out of TMEM (one thread per head),
//     write P (bf16) to shared memory, and rescale the O^T accumulator in TMEM
//     only when a head's running max grows by more than 2^8.
// Partial (O, m, l) per split go to the workspace; decode_combine merges the
// splits with their log-sum-exp weights, normalises, applies the inverse RoPE
// to the rotary channels and stores bf16 or fp32.
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

namespace {

constexpr int kTileRows = 64;
constexpr int kStages = 2;
constexpr int kDim = 512;
constexpr int kChunks = kDim / 64;                 // 64-channel (128-byte) column chunks
constexpr int kChunkBytes = kTileRows * 128;       // 8 KB
constexpr int kTileBytes = kChunks * kChunkBytes;  // 64 KB
constexpr int kQBytes = kChunks * 64 * 128;        // 64 heads x 512 channels, 16-bit
constexpr int kPBytes = 64 * 128;                  // 64 heads x 64 rows, 16-bit
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // O^T: 4 channel tiles x 64 heads
constexpr uint32_t kColS = 256;  // scores: 2 buffers x 64 rows (M = 64 layout)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Per-format configuration.  bf16 caches go straight from HBM to the MMA
// operand tile by TMA gather and run kind::f16 with bf16 inputs.  Quantised
// caches are dequantised in the load path by four converter warps (16-byte
// loads straight from HBM, hardware cvt to f16, swizzled stores); every
// E4M3 value and every E2M1 x E4M3 product is exact in f16, so those run
// kind::f16 with f16 inputs (Q is converted to f16 once per CTA).
template <int FMT>
struct Cfg {
  static constexpr bool kQuant = FMT != DSV4KV_BF16;
  static constexpr bool kRowScale = FMT == DSV4KV_FP8_E4M3_ROW;
  static constexpr int kThreads = kQuant ? 320 : 192;
  static constexpr uint32_t kIdescQK = kQuant ? idesc_f16(64, 64, 0, 0) : idesc_bf16(64, 64, 0, 0);
  static constexpr uint32_t kIdescPV = kQuant ? idesc_f16(128, 64, 1, 0) : idesc_bf16(128, 64, 1, 0);
};

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t q_ready;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_done;
  uint32_t tmem_base;
  volatile int abort;
  float alpha[64];
  float row_scale[kStages][kTileRows];
};

constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kTileBytes + 2 * kPBytes + sizeof(Ctl);

struct Params {
  int heads;
  int64_t n;
  int window;
  int k;
  int comp_tiles, tiles, splits, tiles_per_split;
  int64_t comp_rows, win_rows;  // per-sequence row capacity of each cache
  const int32_t* idx;           // [B][k] or null (dense)
  const uint8_t* comp_codes;    // quantised caches (converter warps)
  const void* comp_scales;
  const uint8_t* win_codes;
  const void* win_scales;
  float score_scale;            // sm_scale * log2(e)
  float* o_part;                // [B][splits][H][512]
  float* ml_part;               // [B][splits][H][4]: (m_o, m_l, l, 0)
  uint32_t* status;
};

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait (about one second); on timeout or when another role gave up,
// returns false and raises the CTA's abort flag.
__device__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (ctl->abort) return false;
    if (globaltimer() - t0 > 1000000000ull) {
      ctl->abort = 1;
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Ctl* ctl, int lane) {
  bool ok = true;
  if (lane == 0) ok = wait_or_abort(bar, parity, ctl);
  return __shfl_sync(kFull, ok, 0);
}

__device__ __forceinline__ bool named_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\tbarrier.cta.red.or.pred po, 1, 128, pi;\n\tselp.u32 "
      "%0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)));
  return r != 0;
}
__device__ __forceinline__ void named_bar_sync() { asm volatile("barrier.cta.sync 1, 128;" ::: "memory"); }

// Source of row `r` of tile T: global row (b * rows + i) of the compressed
// cache (from_win = false) or of the window cache; valid = false for padding
// slots and for rejected indices (the row then reads nothing).
struct RowSrc {
  int64_t row;
  bool valid, from_win;
};
__device__ __forceinline__ RowSrc row_source(const Params& p, int b, int T, int r) {
  RowSrc s{0, false, false};
  if (T < p.comp_tiles) {
    const int slot = T * kTileRows + r;
    int64_t i = -1;
    if (p.idx) {
      const int32_t v = slot < p.k ? p.idx[size_t(b) * p.k + slot] : -1;
      if (v >= p.n) set_status(p.status, DSV4KV_DEV_BAD_INDEX);
      i = v;
    } else if (slot < p.n) {
      i = slot;
    }
    s.valid = i >= 0 && i < p.n;
    s.row = int64_t(b) * p.comp_rows + (s.valid ? i : 0);
  } else {
    const int wr = (T - p.comp_tiles) * kTileRows + r;
    s.from_win = true;
    s.valid = wr < p.window;
    s.row = int64_t(b) * p.win_rows + (s.valid ? wr : 0);
  }
  return s;
}

// Row validity of tile T (rows lane and lane+32 of the tile), warp-wide.
__device__ __forceinline__ uint64_t tile_valid_mask(const Params& p, int b, int T, int lane) {
  bool v0, v1;
  if (T < p.comp_tiles) {
    const int s0 = T * kTileRows + lane, s1 = s0 + 32;
    if (p.idx) {
      const int32_t* ib = p.idx + size_t(b) * p.k;
      const int32_t i0 = s0 < p.k ? ib[s0] : -1, i1 = s1 < p.k ? ib[s1] : -1;
      v0 = i0 >= 0 && i0 < p.n;
      v1 = i1 >= 0 && i1 < p.n;
    } else {
      v0 = s0 < p.n;
      v1 = s1 < p.n;
    }
  } else {
    const int w0 = (T - p.comp_tiles) * kTileRows + lane;
    v0 = w0 < p.window;
    v1 = w0 + 32 < p.window;
  }
  return uint64_t(__ballot_sync(kFull, v0)) | (uint64_t(__ballot_sync(kFull, v1)) << 32);
}

// 2^x with the hardware approximation (max relative error ~2^-22, far below
// the 16-bit rounding of P); ex2(-inf) = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_p(float a, float b, bool f16) {
  return f16 ? f32x2_to_f16x2_sat(a, b) : pack_bf16x2(a, b);
}
__device__ __forceinline__ float p_lo(uint32_t v, bool f16) {
  if (!f16) return bf16lo(v);
  float f;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(f) : "r"(v));
  return f;
}
__device__ __forceinline__ float p_hi(uint32_t v, bool f16) {
  if (!f16) return bf16hi(v);
  float f;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(v));
  return f;
}

template <int FMT>
__global__ void __launch_bounds__(Cfg<FMT>::kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_comp,
                  const __grid_constant__ CUtensorMap tm_win, const Params p) {
  using C = Cfg<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sR = sQ + kQBytes;
  uint8_t* sP = sR + kStages * kTileBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(sP + 2 * kPBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int t0 = split * p.tiles_per_split;
  const int nt = max(0, min(p.tiles, t0 + p.tiles_per_split) - t0);
  pdl_trigger();

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_ready, 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], C::kQuant ? 4 : 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], 4);
      mbar_init(&ctl->p_full[s], 4);
    }
    mbar_init(&ctl->pv_done, 1);
    mbar_init(&ctl->o_done, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    if (!C::kQuant) {
      prefetch_tmap(&tm_comp);
      prefetch_tmap(&tm_win);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  pdl_wait();  // everything above touched only shared memory, TMEM and the tensor maps

  if (warp == 0) {
    // ------------------------------------------------------------ producer (TMA)
    if (lane == 0) {
      mbar_arrive_expect_tx(&ctl->q_full, kQBytes);
      for (int c = 0; c < kChunks; ++c) tma_load_3d(sQ + c * kChunkBytes, &tm_q, &ctl->q_full, c * 64, 0, b);
    }
    int issued = 0;
    if (!C::kQuant) {
      for (int i = 0; i < nt; ++i) {
        const int T = t0 + i, stage = i % kStages;
        if (i >= kStages && !warp_wait(&ctl->empty[stage], ((i / kStages) - 1) & 1, ctl, lane)) break;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->full[stage], kTileBytes);
        __syncwarp();
        const int g = lane & 15;  // 4-row group of this lane
        int32_t r[4];
        bool from_win = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const RowSrc s = row_source(p, b, T, 4 * g + e);
          r[e] = int32_t(s.row);
          from_win = s.from_win;
        }
        const CUtensorMap* tm = from_win ? &tm_win : &tm_comp;
        uint8_t* dst = sR + stage * kTileBytes + g * 512;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = (lane >> 4) * 4 + cc;
          tma_gather4(dst + c * kChunkBytes, tm, &ctl->full[stage], c * 64, r[0], r[1], r[2], r[3]);
        }
        issued = i + 1;
      }
    }
    // drain: never leave the CTA with copies in flight
    if (lane == 0) {
      wait_or_abort(&ctl->q_full, 0, ctl);
      for (int i = max(0, issued - kStages); i < issued; ++i)
        wait_or_abort(&ctl->full[i % kStages], (i / kStages) & 1, ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait_or_abort(C::kQuant ? &ctl->q_ready : &ctl->q_full, 0, ctl);
      const uint32_t q_addr = smem_u32(sQ);
      for (int i = 0; ok && i <= nt; ++i) {
        if (i < nt) {
          const int stage = i % kStages, sb = i & 1;
          ok = wait_or_abort(&ctl->full[stage], (i / kStages) & 1, ctl);
          if (ok && i >= 2) ok = wait_or_abort(&ctl->s_free[sb], ((i - 2) >> 1) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t r_addr = smem_u32(sR + stage * kTileBytes);
          const uint32_t d = tmem + kColS + 64 * sb;
#pragma unroll
          for (int kk = 0; kk < kDim / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
            mma_bf16_ss(d, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(r_addr + off, 16, 1024),
                        C::kIdescQK, kk > 0);
          }
          mma_commit(&ctl->s_full[sb]);
        }
        if (i >= 1) {
          const int j = i - 1, stage = j % kStages, pb = j & 1;
          ok = wait_or_abort(&ctl->p_full[pb], (j >> 1) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t r_addr = smem_u32(sR + stage * kTileBytes);
          const uint32_t p_addr = smem_u32(sP + pb * kPBytes);
#pragma unroll
          for (int ct = 0; ct < kDim / 128; ++ct) {
#pragma unroll
            for (int kr = 0; kr < kTileRows / 16; ++kr) {
              const uint64_t a = smem_desc_sw128(r_addr + 2 * ct * kChunkBytes + kr * 2048, kChunkBytes, 1024);
              const uint64_t bd = smem_desc_sw128(p_addr + kr * 32, 16, 1024);
              mma_bf16_ss(tmem + kColO + 64 * ct, a, bd, C::kIdescPV, (j > 0 || kr > 0) ? 1u : 0u);
            }
          }
          mma_commit(&ctl->empty[stage]);
          mma_commit(&ctl->pv_done);
        }
      }
      mma_commit(&ctl->o_done);  // completes once every issued MMA has finished
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue (warps 2..5)
    // After a timed-out wait a warp turns `dead` (warp-uniform): it skips
    // every wait, TMEM and shared-memory access but still takes part in the
    // group's named barriers, so the other softmax warps cannot hang on them.
    //
    // Two running maxima: m_l for the softmax denominator l and m_o for the
    // weights that multiply the stored rows.  With fp8 rows the per-row scale
    // s_r is folded into the weights (w_r = p_r * s_r, y_r = x_r + log2 s_r),
    // so the accumulator's weights stay <= 2^8 whatever the scales are; for
    // other formats y == x and the two maxima coincide.
    const int wq = warp & 3;  // TMEM lane quadrant of this warp
    const uint32_t lane_base = uint32_t(32 * wq) << 16;
    const bool head_thread = lane < 16;
    const int h = 16 * wq + (lane & 15);
    float m_o = -INFINITY, m_l = -INFINITY, l = 0.f;
    bool dead = false;
    for (int i = 0; i < nt; ++i) {
      const int T = t0 + i, sb = i & 1, stage = i % kStages;
      if (!dead) dead = !warp_wait(&ctl->s_full[sb], (i >> 1) & 1, ctl, lane);
      if (C::kRowScale && !dead) dead = !warp_wait(&ctl->full[stage], (i / kStages) & 1, ctl, lane);
      float x[64];
      float tmax = -INFINITY, ymax = -INFINITY;
      if (!dead) {
        tc_fence_after();
        uint32_t s0[32], s1[32];
        tmem_ld32(tmem + lane_base + kColS + 64 * sb, s0);
        tmem_ld32(tmem + lane_base + kColS + 64 * sb + 32, s1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->s_free[sb]);
        const uint64_t vmask = tile_valid_mask(p, b, T, lane);
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          const float raw = __uint_as_float(r < 32 ? s0[r] : s1[r - 32]);
          const bool v = (vmask >> r) & 1;
          if (C::kRowScale) {
            const float sc = ctl->row_scale[stage][r];
            x[r] = v ? raw * sc * p.score_scale : -INFINITY;
            ymax = fmaxf(ymax, (v && sc > 0.f) ? x[r] + __log2f(sc) : -INFINITY);
          } else {
            x[r] = v ? raw * p.score_scale : -INFINITY;
          }
          tmax = fmaxf(tmax, x[r]);
        }
        if (!C::kRowScale) ymax = tmax;
        if (i >= 1) dead = !warp_wait(&ctl->pv_done, (i - 1) & 1, ctl, lane);
      }
      if (!dead && tmax > m_l + kRescaleThreshold) {
        l *= (m_l == -INFINITY) ? 0.f : exp2f(m_l - tmax);
        m_l = tmax;
      }
      const bool need = !dead && head_thread && ymax > m_o + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m_o == -INFINITY) ? 0.f : exp2f(m_o - ymax);
        m_o = ymax;
      }
      if (i >= 1 && named_bar_or(need)) {
        if (!dead && head_thread) ctl->alpha[h] = alpha;
        named_bar_sync();
        if (!dead) {
          tc_fence_after();
#pragma unroll 1
          for (int ct = 0; ct < kDim / 128; ++ct) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              uint32_t o[32];
              const uint32_t addr = tmem + lane_base + kColO + 64 * ct + 32 * half;
              tmem_ld32(addr, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e)
                o[e] = __float_as_uint(__uint_as_float(o[e]) * ctl->alpha[32 * half + e]);
              tmem_st32(addr, o);
            }
          }
          tmem_wait_st();
        }
        named_bar_sync();  // alpha[] is rewritten only after everyone read it
      }
      if (dead) continue;
      if (head_thread) {
        uint8_t* prow = sP + sb * kPBytes + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 8 * c16 + 2 * e;
            float ya = x[r], yb = x[r + 1];
            if (C::kRowScale) {  // y = x + log2(s_r): the weight of the stored row carries its scale
              const float sa = ctl->row_scale[stage][r], sb2 = ctl->row_scale[stage][r + 1];
              ya = sa > 0.f ? ya + __log2f(sa) : -INFINITY;
              yb = sb2 > 0.f ? yb + __log2f(sb2) : -INFINITY;
            }
            const float wa = (m_o == -INFINITY) ? 0.f : fast_exp2(ya - m_o);
            const float wb = (m_o == -INFINITY) ? 0.f : fast_exp2(yb - m_o);
            const uint32_t packed = pack_p(wa, wb, C::kQuant);
            if (C::kRowScale) {
              if (m_l != -INFINITY) l += fast_exp2(x[r] - m_l) + fast_exp2(x[r + 1] - m_l);
            } else {
              l += p_lo(packed, C::kQuant) + p_hi(packed, C::kQuant);  // the weights the MMA uses
            }
            w[e] = packed;
          }
          *reinterpret_cast<uint4*>(prow + ((c16 ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[sb]);
    }
    if (!dead) dead = !warp_wait(&ctl->o_done, 0, ctl, lane);
    float* ml = p.ml_part + ((size_t(b) * p.splits + split) * p.heads + h) * 4;
    if (!dead) {
      tc_fence_after();
      float* op = p.o_part + (size_t(b) * p.splits + split) * size_t(p.heads) * kDim;
#pragma unroll 1
      for (int ct = 0; ct < kDim / 128; ++ct) {
        const int c = 128 * ct + 32 * wq + lane;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kColO + 64 * ct + 32 * half, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int hh = 32 * half + e;
            if (hh < p.heads) op[size_t(hh) * kDim + c] = __uint_as_float(o[e]);
          }
        }
      }
      if (head_thread && h < p.heads) *reinterpret_cast<float4*>(ml) = make_float4(m_o, m_l, l, 0.f);
    } else if (head_thread && h < p.heads) {
      // an empty partial keeps the combine step finite
      *reinterpret_cast<float4*>(ml) = make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
    }
  } else if (C::kQuant) {
    // ------------------------------------------------------------ converters (warps 6..9)
    const int cw = warp - 6;
    const int tid = threadIdx.x - 192;
    // (1) Q: bf16 -> f16 in place (saturating), once per CTA
    if (warp_wait(&ctl->q_full, 0, ctl, lane)) {
      for (int v = tid; v < kQBytes / 16; v += 128) {
        uint4 x = *reinterpret_cast<const uint4*>(sQ + 16 * v);
        x = make_uint4(f32x2_to_f16x2_sat(bf16lo(x.x), bf16hi(x.x)), f32x2_to_f16x2_sat(bf16lo(x.y), bf16hi(x.y)),
                       f32x2_to_f16x2_sat(bf16lo(x.z), bf16hi(x.z)), f32x2_to_f16x2_sat(bf16lo(x.w), bf16hi(x.w)));
        *reinterpret_cast<uint4*>(sQ + 16 * v) = x;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->q_ready);
    }
    // (2) rows: warp cw converts rows 16*cw .. 16*cw+15 of every tile; lane
    // `lane` owns channels [16*lane, 16*lane+16) = half of a 64-channel chunk.
    const int chunk = lane >> 2, u0 = (lane & 3) * 2;
    for (int i = 0; i < nt; ++i) {
      const int T = t0 + i, stage = i % kStages;
      if (i >= kStages && !warp_wait(&ctl->empty[stage], ((i / kStages) - 1) & 1, ctl, lane)) break;
      // lane j < 16 resolves row 16*cw + j, then every lane reads all 16 answers
      const RowSrc mine = row_source(p, b, T, 16 * cw + (lane & 15));
      const bool from_win = mine.from_win;  // uniform within a tile
      const uint8_t* codes = from_win ? p.win_codes : p.comp_codes;
      const void* scales = from_win ? p.win_scales : p.comp_scales;
      if (C::kRowScale && lane < 16)
        ctl->row_scale[stage][16 * cw + lane] = mine.valid ? static_cast<const float*>(scales)[mine.row] : 0.f;
      uint4 raw[16];
      uint32_t sgrp[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int64_t row = __shfl_sync(kFull, mine.row, j);
        const bool valid = __shfl_sync(kFull, mine.valid, j);
        if (C::kRowScale) {
          raw[j] = valid ? ld_stream_v4(codes + size_t(row) * kDim + 16 * lane) : make_uint4(0, 0, 0, 0);
          sgrp[j] = 0;
        } else {
          if (valid) {
            const uint2 c8 = *reinterpret_cast<const uint2*>(codes + size_t(row) * (kDim / 2) + 8 * lane);
            raw[j] = make_uint4(c8.x, c8.y, 0, 0);
            sgrp[j] = static_cast<const uint8_t*>(scales)[size_t(row) * (kDim / 16) + lane];
          } else {
            raw[j] = make_uint4(0, 0, 0, 0);
            sgrp[j] = 0;
          }
        }
      }
      uint8_t* tile = sR + stage * kTileBytes + chunk * kChunkBytes;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = 16 * cw + j;
        uint32_t hv[8];
        if (C::kRowScale) {
          const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            hv[2 * e] = e4m3x2_to_f16x2(w[e] & 0xffffu);
            hv[2 * e + 1] = e4m3x2_to_f16x2(w[e] >> 16);
          }
        } else {
          const uint32_t s2 = e4m3x2_to_f16x2(sgrp[j] | (sgrp[j] << 8));  // (scale, scale) as f16x2
          const uint32_t w[2] = {raw[j].x, raw[j].y};
#pragma unroll
          for (int e = 0; e < 8; ++e) hv[e] = hmul2(e2m1x2_to_f16x2((w[e >> 2] >> (8 * (e & 3))) & 0xffu), s2);
        }
        uint8_t* line = tile + r * 128;
        *reinterpret_cast<uint4*>(line + ((u0 ^ (r & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(line + (((u0 + 1) ^ (r & 7)) << 4)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->full[stage]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && ctl->abort) set_status(p.status, DSV4KV_DEV_TIMEOUT);
}

// Merge split partials, normalise, inverse RoPE.  Per split: O_s (weights
// relative to 2^m_o), l_s (relative to 2^m_l):
//   out = [sum_s O_s 2^(m_o,s - Mo)] / [sum_s l_s 2^(m_l,s - Ml)] * 2^(Mo - Ml).
__global__ void __launch_bounds__(128) decode_combine(const float* __restrict__ o_part,
                                                      const float* __restrict__ ml_part, int splits, int heads,
                                                      int64_t t, int rope_dim, double rope_base, int out_fp32,
                                                      void* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.x;
  const int b = bh / heads, h = bh % heads;
  const int c = 4 * threadIdx.x;
  float Mo = -INFINITY, Ml = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const float4 ml = *reinterpret_cast<const float4*>(ml_part + ((size_t(b) * splits + s) * heads + h) * 4);
    Mo = fmaxf(Mo, ml.x);
    Ml = fmaxf(Ml, ml.y);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const float4 ml = *reinterpret_cast<const float4*>(ml_part + ((size_t(b) * splits + s) * heads + h) * 4);
    if (ml.y != -INFINITY) L += ml.z * exp2f(ml.y - Ml);
    if (ml.x == -INFINITY) continue;
    const float w = exp2f(ml.x - Mo);
    const float4 o = *reinterpret_cast<const float4*>(o_part + ((size_t(b) * splits + s) * heads + h) * kDim + c);
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  const float inv = (Mo == -INFINITY) ? 0.f : exp2f(Mo - Ml) / L;
  float v[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  const int r0 = kDim - rope_dim;
  if (c >= r0) {
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int m = (c + e - r0) >> 1;
      // angle -t*theta in units of pi, reduced exactly modulo 2 before sincospi
      const double ang = double(t) * (pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793);
      const double xr = ang - 2.0 * rint(0.5 * ang);
      double sn, cs;
      sincospi(-xr, &sn, &cs);
      const float x = v[e], y = v[e + 1];
      v[e] = float(x * cs - y * sn);
      v[e + 1] = float(x * sn + y * cs);
    }
  }
  const size_t o = (size_t(b) * heads + h) * kDim + c;
  if (out_fp32) {
    *reinterpret_cast<float4*>(static_cast<float*>(out) + o) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + o) =
        make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
  }
}

struct Plan {
  int comp_tiles, tiles, splits, tiles_per_split;
};

Plan make_plan(int batch, int comp_tiles, int win_tiles) {
  Plan pl{};
  pl.comp_tiles = comp_tiles;
  pl.tiles = comp_tiles + win_tiles;
  const int sms = sm_count();
  // one CTA per SM at most (shared memory), so at most one wave
  int splits = std::max(1, std::min(pl.tiles, sms / std::max(batch, 1)));
  pl.tiles_per_split = (pl.tiles + splits - 1) / splits;
  pl.splits = (pl.tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
  return pl;
}

struct DecodeWs {
  uint32_t* status;
  float* o_part;
  float* ml_part;
  size_t bytes;
};

DecodeWs decode_ws_layout(char* base, int batch, int heads, const Plan& pl) {
  DecodeWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = (off + bytes + 255) / 256 * 256;
    return p;
  };
  w.status = reinterpret_cast<uint32_t*>(take(16));
  w.o_part = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * pl.splits * heads * kDim));
  w.ml_part = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * pl.splits * heads * 4));
  w.bytes = off;
  return w;
}

}  // namespace

size_t decode_ws_bytes(int batch, int heads, int dim, int64_t rows_per_seq) {
  (void)dim;
  // rows_per_seq = compressed slots + window rows; the split plan only depends on the tile count
  const int tiles = int((rows_per_seq + kTileRows - 1) / kTileRows) + 1;
  Plan pl{};
  pl.splits = std::max(1, std::min(tiles, sm_count() / std::max(batch, 1)));  // upper bound of make_plan
  return decode_ws_layout(nullptr, batch, heads, pl).bytes;
}

template <int FMT>
dsv4kv_status launch_fmt(const CUtensorMap& tq, const CUtensorMap& tc, const CUtensorMap& tw, const Params& p,
                         int grid, cudaStream_t stream) {
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    if (cudaFuncSetAttribute(decode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes)) !=
        cudaSuccess)
      return check_launch("decode: cudaFuncSetAttribute");
    attr_set = true;
  }
  launch_pdl(decode_kernel<FMT>, dim3(grid), dim3(Cfg<FMT>::kThreads), kSmemBytes, stream, tq, tc, tw, p);
  return check_launch("decode_kernel");
}

dsv4kv_status decode_launch(const DecodeArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (a.dim != kDim) return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: dim must be 512 (got %d)", a.dim);
  const int fmt = a.comp.fmt;
  if (a.win.fmt != fmt)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: the window cache must have the compressed cache's format");
  if (fmt != DSV4KV_BF16 && fmt != DSV4KV_FP8_E4M3_ROW && fmt != DSV4KV_FP4_E2M1_G16)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: unknown cache format %d", fmt);
  const int slots = a.idx ? a.k : int(a.n);
  const int comp_tiles = (a.n > 0 && slots > 0) ? (slots + kTileRows - 1) / kTileRows : 0;
  const int win_tiles = (a.window + kTileRows - 1) / kTileRows;
  if (comp_tiles + win_tiles == 0) return set_error(DSV4KV_ERR_INVALID_ARG, "decode: no rows to attend");
  const Plan pl = make_plan(a.batch, comp_tiles, win_tiles);
  const DecodeWs w = decode_ws_layout(static_cast<char*>(ws), a.batch, a.heads, pl);
  if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "decode: workspace too small");

  CUtensorMap tq, tc, tw;
  if (!encode_tmap_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, kDim, uint64_t(a.heads), uint64_t(a.batch),
                      uint64_t(kDim) * 2, uint64_t(a.heads) * kDim * 2, 64, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the query tensor map");
  const dsv4kv_cache& cc = a.comp;
  if (fmt == DSV4KV_BF16) {
    // row gathers (box: 64 channels x 1 row, 128-byte swizzle)
    const void* comp_base = cc.codes ? cc.codes : a.win.codes;
    const uint64_t comp_rows_total = std::max<uint64_t>(1, uint64_t(a.batch) * uint64_t(std::max<int64_t>(cc.rows, 1)));
    if (!encode_tmap_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, comp_base, kDim, comp_rows_total, uint64_t(kDim) * 2,
                        64, 1, CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the compressed-cache tensor map");
    const void* win_base = a.win.codes ? a.win.codes : comp_base;
    const uint64_t win_rows_total = std::max<uint64_t>(1, uint64_t(a.batch) * uint64_t(std::max<int64_t>(a.win.rows, 1)));
    if (!encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, win_base, kDim, win_rows_total, uint64_t(kDim) * 2, 64,
                        1, CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the window tensor map");
  } else {
    tc = tq;  // unused: quantised rows are loaded by the converter warps
    tw = tq;
  }

  Params p{};
  p.heads = a.heads;
  p.n = a.n;
  p.window = a.window;
  p.k = a.idx ? a.k : 0;
  p.comp_tiles = pl.comp_tiles;
  p.tiles = pl.tiles;
  p.splits = pl.splits;
  p.tiles_per_split = pl.tiles_per_split;
  p.comp_rows = cc.rows;
  p.win_rows = a.win.rows;
  p.idx = a.idx;
  p.comp_codes = static_cast<const uint8_t*>(cc.codes);
  p.comp_scales = cc.scales;
  p.win_codes = static_cast<const uint8_t*>(a.win.codes);
  p.win_scales = a.win.scales;
  p.score_scale = a.sm_scale * 1.4426950408889634f;
  p.o_part = w.o_part;
  p.ml_part = w.ml_part;
  p.status = w.status;

  const int grid = a.batch * pl.splits;
  dsv4kv_status st;
  switch (fmt) {
    case DSV4KV_BF16: st = launch_fmt<DSV4KV_BF16>(tq, tc, tw, p, grid, stream); break;
    case DSV4KV_FP8_E4M3_ROW: st = launch_fmt<DSV4KV_FP8_E4M3_ROW>(tq, tc, tw, p, grid, stream); break;
    default: st = launch_fmt<DSV4KV_FP4_E2M1_G16>(tq, tc, tw, p, grid, stream); break;
  }
  if (st != DSV4KV_OK) return st;
  launch_pdl(decode_combine, dim3(a.batch * a.heads), dim3(kDim / 4), 0, stream, (const float*)w.o_part,
             (const float*)w.ml_part, pl.splits, a.heads, a.t, a.rope_dim, a.rope_base, a.out_fp32, a.out);
  return check_launch("decode_combine");
}

}  // namespace dsv4kv
