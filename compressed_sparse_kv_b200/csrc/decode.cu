// Shared-K/V decode attention over compressed entries plus the window.
//
// [P2] Step 3: one cached vector S_j serves as the key (score = Q . S_j) and
// as the value; [P1] "The sliding window": every layer also reads 128 exact
// recent rows; [P1] "Shared key and value": an inverse RoPE is applied to the
// output; [P1] "c4a" / "c128a" and [P2] Step 5: c4a reads the top-k selected
// entries, c128a reads all of them.
//
// One CTA per (sequence, split) walks a contiguous range of 64-row tiles of
// the sequence's row list (selected or all compressed rows, then the window
// rows).  Roles (10 warps):
//   * warp 0 loads Q (one 4-D TMA box, 128-byte swizzle) and every tile whose
//     rows are contiguous in HBM (dense compressed rows, window rows) as one
//     3-D TMA box of 64 rows x 8 chunks of 64 channels;
//   * warps 6-9 load the tiles that are not: gathered bf16 rows with 16-byte
//     cp.async straight into the swizzled tile (each lane reading its row's
//     index from the selection), and quantised rows (fp8 / fp4) with 16-byte
//     loads one tile ahead and hardware cvt to f16 (exact);
//   * warp 1 (one thread) issues tcgen05.mma: S = Q . R^T (M = 64 heads,
//     N = 64 rows, 32 K-steps of 16 channels; head h lands in TMEM lane
//     32*(h/16) + h%16, row r in column r), and O^T += R^T . P^T
//     (M = 128 channels x 4, N = 64 heads, K = 64 rows) from the SAME
//     shared-memory tile — the shared-K/V saving.  It issues whichever
//     product is ready first;
//   * warps 2-5 run the online softmax out of TMEM with 16-lane loads: a
//     quad of threads shares two heads, each thread 16 rows of both; they
//     write P (16-bit) to shared memory and rescale the O^T accumulator in
//     TMEM only when a head's running max grows by > 2^8.
// With one split per sequence the CTA normalises, applies the inverse RoPE
// and stores the output itself; otherwise partial (O, m, l) go to the
// workspace (O as bf16) and decode_combine merges them with log-sum-exp
// weights (or, when enabled, the splits of a thread-block cluster merge over
// distributed shared memory: cluster_merge).  TMEM is freed after every
// warp has arrived on a retire barrier.
#include <cmath>
#include <cstdint>
#include <cstdlib>

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
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // O^T: 4 channel tiles x 64 heads
constexpr uint32_t kColS = 256;  // scores: 2 buffers x 64 columns
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Per-format configuration.  bf16 rows feed kind::f16 MMAs with bf16 inputs.
// Quantised rows are dequantised in the load path; every E4M3 value and every
// E2M1 x E4M3 product is exact in f16, so those run kind::f16 with f16 inputs
// (Q is converted to f16 once per CTA).
template <int FMT>
struct Cfg {
  static constexpr bool kQuant = FMT != DSV4KV_BF16;
  static constexpr bool kRowScale = FMT == DSV4KV_FP8_E4M3_ROW || FMT == DSV4KV_FP8_E4M3_ROW_ROPE_BF16;
  static constexpr uint32_t kIdescQK = kQuant ? idesc_f16(64, 64, 0, 0) : idesc_bf16(64, 64, 0, 0);
  static constexpr uint32_t kIdescPV = kQuant ? idesc_f16(128, 64, 1, 0) : idesc_bf16(128, 64, 1, 0);
};

struct __align__(16) Ctl {
  uint64_t q_full;
  uint64_t q_ready;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];  // PV of the tiles that used P buffer 0 / 1
  uint64_t o_done;
  uint64_t retire;  // one arrival per warp once it is done with TMEM and shared memory
  uint32_t tmem_base;
  volatile int abort;
  float alpha[64];
  float fin[64];
  float row_scale[kStages][kTileRows];
  float row_ls[kStages][kTileRows];   // log2 of the row scale (-inf: no row)
  float row_inv[kStages][kTileRows];  // 1 / row scale (0: no row)
  uint32_t vmask[kStages][4];  // row validity of a gathered tile, 16 rows per loader warp
  float rope_cs[kDim / 2];  // inverse-RoPE rotation of pair m: cos / sin of -t * theta_m
  float rope_sn[kDim / 2];
  // in-cluster merge: this split's (m_o, m_l, l) per head, read by every CTA
  // of the cluster; the merged statistics; this split's weight per head
  float4 st[64];
  float4 gst[64];
  float a_self[64];
};

constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kTileBytes + 2 * kPBytes + sizeof(Ctl);
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// Where the rows of one cache live: a dense [B][rows] layout (table null:
// row i of sequence b is row b * rows + i) or pages of a shared pool (row i
// of sequence b is pool row table[b * tstride + i / page] * page + i % page).
struct RowMap {
  const int32_t* table;
  int page, tstride;
  int64_t rows;   // dense: rows per sequence; paged: rows in the pool
  int64_t pages;  // paged: pages in the pool
};

struct Params {
  int heads;
  int64_t n;    // compressed entries (uniform batch) or the most any sequence has (ragged)
  int window;   // window rows (uniform) or the window length W (ragged)
  int k;
  int splits;
  const int64_t* t_seq;  // ragged batch: query position of every sequence; null = uniform
  int64_t t_max;
  int stride;
  RowMap comp_map, win_map;
  const int32_t* idx;           // [B][k] or null (dense)
  const uint8_t* comp_codes;
  const void* comp_scales;
  const uint8_t* win_codes;
  const void* win_scales;
  float score_scale;  // sm_scale * log2(e)
  uint16_t* o_part;   // [B][splits][H][512] bf16 (the split's unnormalised output)
  float* ml_part;     // [B][splits][H][4]: (m_o, m_l, l, 0)
  float* rope_tab;    // [B][2][256]: the rotation tables for decode_combine (written by split 0)
  int cluster;        // CTAs per thread-block cluster (consecutive splits), merged in the kernel; 1 = none
  uint32_t* status;
  // direct output when splits == 1
  int64_t t;
  int rope_dim;
  double rope_base;
  int out_fp32;
  void* out;
};

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // one second

// Bounded wait; on timeout or when another role gave up, returns false and
// raises the CTA's abort flag.
__device__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (ctl->abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      ctl->abort = 1;
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
// The retire wait: unlike wait_or_abort it does not stop at the abort flag
// (every other wait is bounded, so every warp arrives in the end); it gives
// up only after twice the per-wait limit, and TMEM is freed either way.
__device__ void retire_wait(uint64_t* bar) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, 0))
    if (globaltimer() - t0 > 2 * kWaitLimitNs) return;
}

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

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// The extent of one sequence and the tiles of one CTA.  Tiles 0 ..
// comp_tiles-1 hold the sequence's compressed rows (selected slots or all
// entries, 64 per tile), the rest its window rows.
struct Seq {
  int64_t t, n;  // query position, compressed entries
  int w;         // window rows
  int comp_tiles, tiles, t0, nt;
};

__device__ __forceinline__ Seq seq_info(const Params& p, int b, int split) {
  Seq q;
  if (p.t_seq) {
    int64_t t = p.t_seq[b];
    if (t < 0 || t > p.t_max) {
      set_status(p.status, DSV4KV_DEV_BAD_LENGTH);
      t = t < 0 ? 0 : p.t_max;
    }
    q.t = t;
    q.n = t > p.window ? min(p.n, (t - p.window) / p.stride) : 0;
    q.w = int(t < int64_t(p.window) ? t : int64_t(p.window));
  } else {
    q.t = p.t;
    q.n = p.n;
    q.w = p.window;
  }
  const int64_t slots = p.idx ? (int64_t(p.k) < q.n ? int64_t(p.k) : q.n) : q.n;
  q.comp_tiles = int((slots + kTileRows - 1) / kTileRows);
  q.tiles = q.comp_tiles + (q.w + kTileRows - 1) / kTileRows;
  const int per = (q.tiles + p.splits - 1) / p.splits;
  q.t0 = split * per;
  q.nt = max(0, min(q.tiles, q.t0 + per) - q.t0);
  return q;
}

// Global row of logical row i of sequence b; ok = false (and row 0) when its
// page number is outside the pool.
__device__ __forceinline__ int64_t map_row(const RowMap& m, int b, int64_t i, bool& ok, uint32_t* status) {
  if (!m.table) return int64_t(b) * m.rows + i;
  const int32_t pg = __ldg(m.table + size_t(b) * m.tstride + size_t(i / m.page));
  if (pg < 0 || pg >= m.pages) {
    set_status(status, DSV4KV_DEV_BAD_PAGE);
    ok = false;
    return 0;
  }
  return int64_t(pg) * m.page + i % m.page;
}

// Rows of tile T that exist: the first n - 64T compressed rows (dense) or
// w - 64(T - comp_tiles) window rows.
__device__ __forceinline__ int64_t tile_rows(const Seq& q, int T) {
  return T < q.comp_tiles ? q.n - int64_t(T) * kTileRows : int64_t(q.w) - int64_t(T - q.comp_tiles) * kTileRows;
}

// Whether tile T is loaded by TMA: 64 rows that exist and lie consecutively
// in memory (dense compressed rows or window rows; a page holds whole tiles,
// and its page number is in the pool).  Partial tiles, tiles of bad pages and
// gathered (selected) rows go through the loader warps, which zero-fill what
// does not exist, so no row past a sequence's end is read.
__device__ __forceinline__ bool tile_tma(const Params& p, const Seq& q, int b, int T) {
  if (!((T >= q.comp_tiles || p.idx == nullptr) && tile_rows(q, T) >= kTileRows)) return false;
  const bool win = T >= q.comp_tiles;
  const RowMap& m = win ? p.win_map : p.comp_map;
  if (!m.table) return true;
  const int64_t i0 = int64_t(win ? T - q.comp_tiles : T) * kTileRows;
  const int32_t pg = __ldg(m.table + size_t(b) * m.tstride + size_t(i0 / m.page));
  return pg >= 0 && pg < m.pages;
}

// Source of row `r` of tile T: global row of the compressed cache (from_win =
// false) or of the window cache; valid = false for padding slots, rejected
// indices and rows of bad pages (such rows are zero-filled and masked).
struct RowSrc {
  int64_t row;
  bool valid, from_win;
};
__device__ __forceinline__ RowSrc row_source(const Params& p, const Seq& q, int b, int T, int r) {
  RowSrc s{0, false, false};
  if (T < q.comp_tiles) {
    const int slot = T * kTileRows + r;
    int64_t i = -1;
    if (p.idx) {
      const int32_t v = slot >= p.k ? -1 : __ldg(p.idx + size_t(b) * p.k + slot);
      if (v >= q.n) set_status(p.status, DSV4KV_DEV_BAD_INDEX);
      i = v;
    } else if (slot < q.n) {
      i = slot;
    }
    s.valid = i >= 0 && i < q.n;
    if (s.valid) s.row = map_row(p.comp_map, b, i, s.valid, p.status);
  } else {
    const int wr = (T - q.comp_tiles) * kTileRows + r;
    s.from_win = true;
    s.valid = wr < q.w;
    if (s.valid) s.row = map_row(p.win_map, b, wr, s.valid, p.status);
  }
  return s;
}

// cos / sin of the inverse-RoPE angle -t * rope_base^(-2m/rope_dim): the
// angle in units of pi is reduced exactly modulo 2 before sincospi.
__device__ __forceinline__ void inv_rope_rotation(int64_t t, int m, int rope_dim, double rope_base, float* cs,
                                                  float* sn) {
  const double ang = double(t) * (pow(rope_base, -2.0 * double(m) / double(rope_dim)) / 3.141592653589793);
  double sd, cd;
  sincospi(-(ang - 2.0 * rint(0.5 * ang)), &sd, &cd);
  *cs = float(cd);
  *sn = float(sd);
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

// Writes channel tiles [ct0, ct1) of the CTA's partial O^T (TMEM lanes of
// quarter wq, i.e. channels 128ct + 32wq + lane) to o_part, heads as rows.
// The epilogue warps and the loader warps that share a lane quarter each
// write half of the channel tiles.
__device__ __forceinline__ void store_partial(const Params& p, int b, int split, uint32_t tmem, int wq, int lane,
                                              int ct0, int ct1) {
  const uint32_t lane_base = uint32_t(32 * wq) << 16;
  uint16_t* op = p.o_part + (size_t(b) * p.splits + split) * size_t(p.heads) * kDim;
#pragma unroll 1
  for (int ct = ct0; ct < ct1; ++ct) {
    const int c = 128 * ct + 32 * wq + lane;
    uint32_t o[2][32];  // both halves of the channel tile's 64 heads behind one wait
    tmem_ld32(tmem + lane_base + kColO + 64 * ct, o[0]);
    tmem_ld32(tmem + lane_base + kColO + 64 * ct + 32, o[1]);
    tmem_wait_ld();
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int hh = 32 * half + e;
        if (hh < p.heads) op[size_t(hh) * kDim + c] = f2bf(__uint_as_float(o[half][e]));
      }
  }
}

// The loader warps' part of one quantised tile: warp lw owns rows 16 lw ..
// 16 lw + 15.  fetch() resolves the rows and issues every global load of the
// warp's part into registers; put() (once the stage is free) stores the row
// mask and scales and the rows dequantised to f16 into the 128-byte-swizzled
// tile.  The loaders fetch tile i + 1 right after putting tile i, so its
// loads are in flight while the stage it needs is still in use.
template <int FMT>
struct QuantLoad {
  static constexpr bool kRowScale = Cfg<FMT>::kRowScale;
  static constexpr bool kRope = FMT == DSV4KV_FP8_E4M3_ROW_ROPE_BF16;
  // fp8 rows with bf16 rotary channels: rows of kDim + 64 bytes, 28 chunks of
  // 16 fp8 channels then 8 chunks of 8 bf16 rotary channels; the warp's 16
  // rows hold 448 fp8 chunks (14 per lane) and 128 rotary chunks (4 per lane)
  static constexpr int kBodyChunks = (kDim - 64) / 16, kRopeChunks = 64 / 8;
  static constexpr int kPerBody = 16 * kBodyChunks / 32, kPerRope = 16 * kRopeChunks / 32;
  static constexpr int kRaw = kRope ? kPerBody + kPerRope : 16;
  uint4 raw[kRaw];
  uint32_t sgrp[16];  // fp4: the E4M3 scale of this lane's 16-channel group, per row
  float my_scale;     // row-scale formats: the scale of row 16 lw + lane (lanes < 16)
  uint32_t vb;        // rows of the warp's part that exist

  __device__ __forceinline__ void fetch(const Params& p, const Seq& q, int b, int T, int lw, int lane) {
    const RowSrc mine = row_source(p, q, b, T, 16 * lw + (lane & 15));
    vb = __ballot_sync(kFull, mine.valid) & 0xffffu;
    const uint8_t* codes = mine.from_win ? p.win_codes : p.comp_codes;
    const void* scales = mine.from_win ? p.win_scales : p.comp_scales;
    my_scale = 0.f;
    if (kRowScale && lane < 16 && mine.valid) my_scale = static_cast<const float*>(scales)[mine.row];
    if constexpr (kRope) {
#pragma unroll
      for (int i = 0; i < kPerBody; ++i) {
        const int g = lane + 32 * i, jr = g / kBodyChunks, cr = g % kBodyChunks;
        const int64_t row = __shfl_sync(kFull, mine.row, jr);
        raw[i] = (vb >> jr) & 1u ? ld_stream_v4(codes + size_t(row) * (kDim + 64) + 16 * cr) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kPerRope; ++i) {
        const int g = lane + 32 * i, jr = g / kRopeChunks, cr = g % kRopeChunks;
        const int64_t row = __shfl_sync(kFull, mine.row, jr);
        raw[kPerBody + i] = (vb >> jr) & 1u ? ld_stream_v4(codes + size_t(row) * (kDim + 64) + (kDim - 64) + 16 * cr)
                                            : make_uint4(0, 0, 0, 0);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int64_t row = __shfl_sync(kFull, mine.row, j);
        const bool valid = (vb >> j) & 1u;
        if (kRowScale) {  // lane owns channels [16 lane, 16 lane + 16)
          raw[j] = valid ? ld_stream_v4(codes + size_t(row) * kDim + 16 * lane) : make_uint4(0, 0, 0, 0);
        } else if (valid) {
          const uint2 c8 = *reinterpret_cast<const uint2*>(codes + size_t(row) * (kDim / 2) + 8 * lane);
          raw[j] = make_uint4(c8.x, c8.y, 0, 0);
          sgrp[j] = static_cast<const uint8_t*>(scales)[size_t(row) * (kDim / 16) + lane];
        } else {
          raw[j] = make_uint4(0, 0, 0, 0);
          sgrp[j] = 0;
        }
      }
    }
  }

  __device__ __forceinline__ void put(Ctl* ctl, int stage, uint8_t* tile, int lw, int lane) const {
    if (lane == 0) ctl->vmask[stage][lw] = vb;
    if (kRowScale && lane < 16) {
      const float sr = my_scale;
      ctl->row_scale[stage][16 * lw + lane] = sr;
      ctl->row_ls[stage][16 * lw + lane] = sr > 0.f ? __log2f(sr) : -INFINITY;
      ctl->row_inv[stage][16 * lw + lane] = sr > 0.f ? __frcp_rn(sr) : 0.f;
    }
    if constexpr (kRope) {
      // one conversion loop per chunk kind for the whole warp; the rotary
      // channels are stored as f16 of value / scale so that the row scale
      // folds into the softmax weights exactly as for fp8 rows
#pragma unroll
      for (int i = 0; i < kPerBody; ++i) {
        const int g = lane + 32 * i, jr = g / kBodyChunks, cr = g % kBodyChunks;
        const int r = 16 * lw + jr, ch = 16 * cr, u = (ch & 63) >> 3;
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
        uint32_t hv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hv[2 * e] = e4m3x2_to_f16x2(w[e] & 0xffffu);
          hv[2 * e + 1] = e4m3x2_to_f16x2(w[e] >> 16);
        }
        uint8_t* line = tile + (ch >> 6) * kChunkBytes + r * 128;
        *reinterpret_cast<uint4*>(line + ((u ^ (r & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(line + (((u + 1) ^ (r & 7)) << 4)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
#pragma unroll
      for (int i = 0; i < kPerRope; ++i) {
        const int g = lane + 32 * i, jr = g / kRopeChunks, cr = g % kRopeChunks;
        const int r = 16 * lw + jr, ch = (kDim - 64) + 8 * cr, u = (ch & 63) >> 3;
        const float sr = __shfl_sync(kFull, my_scale, jr);
        const float inv = sr > 0.f ? __frcp_rn(sr) : 0.f;
        const uint4 x = raw[kPerBody + i];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t hv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) hv[e] = f32x2_to_f16x2_sat(bf16lo(w[e]) * inv, bf16hi(w[e]) * inv);
        uint8_t* line = tile + (ch >> 6) * kChunkBytes + r * 128;
        *reinterpret_cast<uint4*>(line + ((u ^ (r & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
    } else {
      const int chunk = lane >> 2, u0 = (lane & 3) * 2;  // lane owns channels [16 lane, 16 lane + 16)
      uint8_t* ctile = tile + chunk * kChunkBytes;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = 16 * lw + j;
        uint32_t hv[8];
        if (kRowScale) {
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
        uint8_t* line = ctile + r * 128;
        *reinterpret_cast<uint4*>(line + ((u0 ^ (r & 7)) << 4)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(line + (((u0 + 1) ^ (r & 7)) << 4)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
    }
  }
};

// In-cluster merge of a sequence's splits.  The C CTAs of a cluster (C a
// power of two <= 16) hold consecutive splits; each holds its unnormalised
// O^T in TMEM and its per-head (m_o, m_l, l) in ctl->st.  The 512 channels
// form 16 units of 32 (channel tile ct, lane quarter wq; unit 4 ct + wq) and
// CTA r owns units [16 r / C, 16 (r + 1) / C).  After a cluster barrier
// (every split's statistics are final and every CTA is done with its tiles,
// whose shared memory becomes the receive buffer) each CTA forms the merged
// statistics, scales its O^T by its weight 2^(m_o - M_o) and stores every
// unit it does not own into the owner's buffer (distributed shared memory,
// 16-byte stores); after a second barrier each owner adds its own TMEM part
// to what it received.  When the cluster spans all splits the owner
// normalises (2^(M_o - M_l) / L), applies the inverse RoPE and writes the
// output; otherwise it writes one merged partial per cluster (group) for
// decode_combine.  Receive buffer (floats): [sender][unit][head / 4][32
// channels][4 heads], 8 KB per (sender, unit), 128 KB in all.
__device__ __forceinline__ void named_bar_sync_256() { asm volatile("barrier.cta.sync 2, 256;" ::: "memory"); }

__device__ __forceinline__ void cluster_merge(const Params& p, const Seq& sq, Ctl* ctl, float* buf, uint32_t tmem, int b,
                                           int split, int warp, int lane) {
  const int C = p.cluster, U = 16 / C;
  const int self = int(cluster_rank());
  const bool final_out = C == p.splits;
  // 1) every CTA's statistics are published and its tiles consumed
  __syncwarp();
  cluster_arrive_release_div();
  cluster_wait_acquire_div();
  // this CTA has an accumulator (it ran tiles, and no wait gave up)
  const bool own = sq.nt > 0 && !ctl->abort;
  if (warp >= 2) {
    tc_fence_after();
    if (warp < 4) {  // one thread per head: the merged statistics
      const int h = threadIdx.x - 64;
      // running (M_o, M_l, L) over the splits' terms (L relative to 2^M_l)
      float mo = -INFINITY, ml = -INFINITY, L = 0.f, mine = -INFINITY;
#pragma unroll 1
      for (int r = 0; r < C; ++r) {
        const float4 v = ld_dsmem_f4(dsmem_addr(&ctl->st[h], uint32_t(r)));
        mo = fmaxf(mo, v.x);
        if (r == self) mine = v.x;
        if (v.y != -INFINITY) {
          if (v.y > ml) {
            L = (ml == -INFINITY ? 0.f : L * fast_exp2(ml - v.y)) + v.z;
            ml = v.y;
          } else {
            L += v.z * fast_exp2(v.y - ml);
          }
        }
      }
      ctl->a_self[h] = (own && mine != -INFINITY) ? fast_exp2(mine - mo) : 0.f;
      ctl->fin[h] = (mo == -INFINITY || !(L > 0.f)) ? 0.f : fast_exp2(mo - ml) / L;
      ctl->gst[h] = make_float4(mo, ml, L, 0.f);
    }
    named_bar_sync_256();
    // 2) scaled O^T of the units this CTA does not own, to their owners
    const int wq = warp & 3, half = warp >= 6 ? 1 : 0;
    const uint32_t lane_base = uint32_t(32 * wq) << 16;
#pragma unroll 1
    for (int ct = 0; ct < kDim / 128; ++ct) {
      const int u = 4 * ct + wq, owner = u / U;
      if (owner == self) continue;
      uint32_t o[32];
      if (own) {
        tmem_ld32(tmem + lane_base + kColO + 64 * ct + 32 * half, o);
        tmem_wait_ld();
      }
      const uint32_t dst =
          dsmem_addr(buf + size_t((self * U + (u - owner * U)) * 16 + 8 * half) * 128 + 4 * lane, uint32_t(owner));
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = ctl->a_self[32 * half + 4 * q + k];
          w[k] = (own && a != 0.f) ? __uint_as_float(o[4 * q + k]) * a : 0.f;
        }
        st_dsmem_f4(dst + uint32_t(q) * 512u, make_float4(w[0], w[1], w[2], w[3]));
      }
    }
  }
  // 3) every contribution is in its owner's buffer
  __syncwarp();
  cluster_arrive_release_div();
  cluster_wait_acquire_div();
  if (warp < 2) return;
  const int wq = warp & 3, half = warp >= 6 ? 1 : 0;
  const uint32_t lane_base = uint32_t(32 * wq) << 16;
  const int r0 = kDim - p.rope_dim, groups = p.splits / C, g = split / C;
#pragma unroll 1
  for (int ct = 0; ct < kDim / 128; ++ct) {
    const int u = 4 * ct + wq;
    if (u / U != self) continue;
    const int ul = u - self * U;
    float acc[32];
    {
      uint32_t o[32];
      if (own) {
        tmem_ld32(tmem + lane_base + kColO + 64 * ct + 32 * half, o);
        tmem_wait_ld();
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float a = ctl->a_self[32 * half + e];
        acc[e] = (own && a != 0.f) ? __uint_as_float(o[e]) * a : 0.f;
      }
    }
#pragma unroll 1
    for (int s = 0; s < C; ++s) {
      if (s == self) continue;
      const float* src = buf + size_t((s * U + ul) * 16 + 8 * half) * 128 + 4 * lane;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(src + 128 * q);
        acc[4 * q] += v.x;
        acc[4 * q + 1] += v.y;
        acc[4 * q + 2] += v.z;
        acc[4 * q + 3] += v.w;
      }
    }
    const int c = 128 * ct + 32 * wq + lane;
    if (final_out) {
      const bool rot = c >= r0;
      const float cs = rot ? ctl->rope_cs[(c - r0) >> 1] : 1.f;
      const float sn = rot ? ctl->rope_sn[(c - r0) >> 1] : 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int hh = 32 * half + e;
        const float f = ctl->fin[hh];
        float v = f != 0.f ? acc[e] * f : 0.f;
        const float partner = __shfl_xor_sync(kFull, v, 1);  // channel c ^ 1 of the same head
        if (rot) v = (c & 1) ? partner * sn + v * cs : v * cs - partner * sn;
        if (hh < p.heads) {
          const size_t oi = (size_t(b) * p.heads + hh) * kDim + c;
          if (p.out_fp32) static_cast<float*>(p.out)[oi] = v;
          else static_cast<uint16_t*>(p.out)[oi] = f2bf(v);
        }
      }
    } else {
      uint16_t* op = p.o_part + (size_t(b) * groups + g) * size_t(p.heads) * kDim + c;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int hh = 32 * half + e;
        if (hh < p.heads) op[size_t(hh) * kDim] = f2bf(acc[e]);
      }
    }
  }
  // the group's merged statistics (one CTA writes them)
  if (!final_out && self == 0 && warp >= 2 && warp < 4) {
    const int h = threadIdx.x - 64;
    if (h < p.heads) {
      const float4 gs = ctl->gst[h];
      *reinterpret_cast<float4*>(p.ml_part + ((size_t(b) * groups + g) * p.heads + h) * 4) =
          gs.x == -INFINITY ? make_float4(-INFINITY, -INFINITY, 0.f, 0.f) : gs;
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
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
  pdl_trigger();

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_ready, 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 5);  // warp 0 + the four loader warps, every tile
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], 4);
      mbar_init(&ctl->p_full[s], 4);
    }
    mbar_init(&ctl->pv_done[0], 1);
    mbar_init(&ctl->pv_done[1], 1);
    mbar_init(&ctl->o_done, 1);
    mbar_init(&ctl->retire, kThreads / 32);
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
  const Seq sq = seq_info(p, b, split);  // (the lengths of a ragged batch may come from the previous kernel)
  const int t0 = sq.t0, nt = sq.nt;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA: Q and contiguous tiles
    if (lane == 0) {
      mbar_arrive_expect_tx(&ctl->q_full, kQBytes);
      tma_load_4d(sQ, &tm_q, &ctl->q_full, 0, 0, 0, b);  // all 8 channel chunks in one box
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int T = t0 + i, stage = i % kStages;
        if (i >= kStages && !wait_or_abort(&ctl->empty[stage], ((i / kStages) - 1) & 1, ctl)) break;
        if (!C::kQuant && tile_tma(p, sq, b, T)) {
          const RowSrc s0 = row_source(p, sq, b, T, 0);  // first row of the run
          const CUtensorMap* tm = s0.from_win ? &tm_win : &tm_comp;
          const int32_t row0 = int32_t(s0.row);
          mbar_arrive_expect_tx(&ctl->full[stage], kTileBytes);
          uint8_t* dst = sR + stage * kTileBytes;
          tma_load_3d(dst, tm, &ctl->full[stage], 0, row0, 0);  // 64 rows x all 8 channel chunks
        } else {
          mbar_arrive(&ctl->full[stage]);
        }
        issued = i + 1;
      }
      // drain: never leave the CTA with copies in flight
      wait_or_abort(&ctl->q_full, 0, ctl);
      for (int i = max(0, issued - kStages); i < issued; ++i)
        wait_or_abort(&ctl->full[i % kStages], (i / kStages) & 1, ctl);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait_or_abort(C::kQuant ? &ctl->q_ready : &ctl->q_full, 0, ctl);
      const uint64_t qd = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      int next_qk = 0, next_pv = 0;
      uint64_t idle_since = 0;
      while (ok && next_pv < nt) {
        bool progressed = false;
        // both products are polled with non-blocking tests, so that one that is
        // not ready never holds up the other
        if (next_pv < next_qk && mbar_test_wait(&ctl->p_full[next_pv & 1], (next_pv >> 1) & 1)) {
          const int j = next_pv, stage = j % kStages, pb = j & 1;
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
          mma_commit(&ctl->pv_done[pb]);
          ++next_pv;
          progressed = true;
        } else if (next_qk < nt && next_qk < next_pv + 2) {
          const int i = next_qk, stage = i % kStages, sb = i & 1;
          if (mbar_test_wait(&ctl->full[stage], (i / kStages) & 1) &&
              (i < 2 || mbar_test_wait(&ctl->s_free[sb], ((i - 2) >> 1) & 1))) {
            tc_fence_after();
            const uint64_t rd = smem_desc_sw128(smem_u32(sR + stage * kTileBytes), 16, 1024);
            const uint32_t d = tmem + kColS + 64 * sb;
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk) {
              const uint32_t off16 = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;  // descriptor address units
              mma_bf16_ss(d, qd + off16, rd + off16, C::kIdescQK, kk > 0);
            }
            mma_commit(&ctl->s_full[sb]);
            ++next_qk;
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = 0;
        } else {
          const uint64_t now = globaltimer();
          if (idle_since == 0) idle_since = now;
          if (ctl->abort || now - idle_since > kWaitLimitNs) {
            ctl->abort = 1;
            ok = false;
          }
        }
      }
      mma_commit(&ctl->o_done);  // completes once every issued MMA has finished
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue (warps 2..5)
    // Warp w reads TMEM lane quarter wq = w % 4 (heads 16wq .. 16wq+15).  A
    // 16x256b.x8 load gives thread i the scores of heads hA = 16wq + i/4 and
    // hB = hA + 8 at rows 8j + 2(i%4) + {0, 1} (j < 8): the four threads of a
    // quad share two heads and reduce over the quad.  After a timed-out wait a
    // warp turns `dead` (warp-uniform): it skips every wait, TMEM and
    // shared-memory access but still takes part in the group's named barriers.
    //
    // Two running maxima per head: m_l for the softmax denominator l and m_o
    // for the weights that multiply the stored rows.  With fp8 rows the
    // per-row scale s_r is folded into the weights (w_r = p_r * s_r,
    // y_r = x_r + log2 s_r), so the accumulator's weights stay <= 2^8 whatever
    // the scales are; for other formats y == x and the two maxima coincide.
    const int wq = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t lane_base = uint32_t(32 * wq) << 16;
    const int g = lane >> 2, c2 = lane & 3;
    const int hd[2] = {16 * wq + g, 16 * wq + 8 + g};
    float m_o[2] = {-INFINITY, -INFINITY}, m_l[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool dead = false;
    // the inverse-RoPE table (fp64 angles, ~1 us of dependent double-precision
    // work), while the first tile loads and its QK runs
    for (int m = threadIdx.x - 64; m < p.rope_dim / 2; m += 128) {
      float cs, sn;
      inv_rope_rotation(sq.t, m, p.rope_dim, p.rope_base, &cs, &sn);
      ctl->rope_cs[m] = cs;
      ctl->rope_sn[m] = sn;
      if (p.splits > p.cluster && split == 0) {  // (decode_combine reads it)
        p.rope_tab[size_t(b) * kDim + m] = cs;
        p.rope_tab[size_t(b) * kDim + kDim / 2 + m] = sn;
      }
    }
    for (int i = 0; i < nt; ++i) {
      const int T = t0 + i, sb = i & 1, stage = i % kStages;
      const bool gathered = C::kQuant || !tile_tma(p, sq, b, T);
      if (!dead) dead = !warp_wait(&ctl->s_full[sb], (i >> 1) & 1, ctl, lane);
      // the loaders' row mask and row scales (complete: the MMA already consumed this tile)
      if ((gathered || C::kRowScale) && !dead) dead = !warp_wait(&ctl->full[stage], (i / kStages) & 1, ctl, lane);
      float x[2][16];
      float tmax[2] = {-INFINITY, -INFINITY}, ymax[2] = {-INFINITY, -INFINITY};
      float2 rsc[C::kRowScale ? 8 : 1], rls[C::kRowScale ? 8 : 1], rinv[C::kRowScale ? 8 : 1];
      if (!dead) {
        tc_fence_after();
        uint32_t sc[32];
        tmem_ld_16x256b_x8(tmem + lane_base + kColS + 64 * sb, sc);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->s_free[sb]);
        const uint64_t vm = gathered ? (uint64_t(ctl->vmask[stage][0]) | (uint64_t(ctl->vmask[stage][1]) << 16) |
                                        (uint64_t(ctl->vmask[stage][2]) << 32) | (uint64_t(ctl->vmask[stage][3]) << 48))
                                     : ~0ull;  // a TMA tile: 64 rows that exist
        if (C::kRowScale) {  // this thread's rows 8j + 2 c2 + {0, 1}: their scale terms, up front
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            rsc[j] = *reinterpret_cast<const float2*>(&ctl->row_scale[stage][8 * j + 2 * c2]);
            rls[j] = *reinterpret_cast<const float2*>(&ctl->row_ls[stage][8 * j + 2 * c2]);
            rinv[j] = *reinterpret_cast<const float2*>(&ctl->row_inv[stage][8 * j + 2 * c2]);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 8 * j + 2 * c2 + e;
            const bool v = (vm >> r) & 1;
            float ls = 0.f, rs = 1.f;
            bool sok = true;
            if (C::kRowScale) {
              rs = e ? rsc[j].y : rsc[j].x;
              ls = e ? rls[j].y : rls[j].x;
              sok = rs > 0.f;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              float xv = v ? __uint_as_float(sc[4 * j + 2 * hh + e]) * p.score_scale : -INFINITY;
              if (C::kRowScale) {
                xv = v ? xv * rs : -INFINITY;
                ymax[hh] = fmaxf(ymax[hh], (v && sok) ? xv + ls : -INFINITY);
              }
              x[hh][2 * j + e] = xv;
              tmax[hh] = fmaxf(tmax[hh], xv);
            }
          }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (!C::kRowScale) ymax[hh] = tmax[hh];
#pragma unroll
          for (int o = 1; o <= 2; o <<= 1) {
            tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(kFull, tmax[hh], o));
            if (C::kRowScale) ymax[hh] = fmaxf(ymax[hh], __shfl_xor_sync(kFull, ymax[hh], o));
          }
          if (!C::kRowScale) ymax[hh] = tmax[hh];
        }
      }
      bool need = false;
      float alpha[2] = {1.f, 1.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!dead && tmax[hh] > m_l[hh] + kRescaleThreshold) {
          l[hh] *= (m_l[hh] == -INFINITY) ? 0.f : fast_exp2(m_l[hh] - tmax[hh]);
          m_l[hh] = tmax[hh];
        }
        if (!dead && ymax[hh] > m_o[hh] + kRescaleThreshold) {
          alpha[hh] = (m_o[hh] == -INFINITY) ? 0.f : fast_exp2(m_o[hh] - ymax[hh]);
          m_o[hh] = ymax[hh];
          need = true;
        }
      }
      if (i >= 1 && named_bar_or(need)) {
        // the accumulator is rescaled: PV(i-1) must have finished adding to it
        if (!dead) dead = !warp_wait(&ctl->pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, ctl, lane);
        if (!dead && c2 == 0) {
          ctl->alpha[hd[0]] = alpha[0];
          ctl->alpha[hd[1]] = alpha[1];
        }
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
      // P buffer sb was last read by PV(i-2)
      if (i >= 2 && !dead) dead = !warp_wait(&ctl->pv_done[sb], ((i - 2) >> 1) & 1, ctl, lane);
      if (dead) continue;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = hd[hh];
        uint8_t* prow = sP + sb * kPBytes + (h >> 3) * 1024 + (h & 7) * 128 + 4 * c2;
        // row-scale formats: sum_r w_r / s_r = sum_r 2^(x_r - m_o), so the
        // denominator's terms 2^(x_r - m_l) need no exponential of their own
        float lw_sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float ya = x[hh][2 * j], yb = x[hh][2 * j + 1];
          if (C::kRowScale) {  // y = x + log2(s_r): the weight of the stored row carries its scale
            ya += rls[j].x;
            yb += rls[j].y;
          }
          const float wa = (m_o[hh] == -INFINITY) ? 0.f : fast_exp2(ya - m_o[hh]);
          const float wb = (m_o[hh] == -INFINITY) ? 0.f : fast_exp2(yb - m_o[hh]);
          const uint32_t packed = pack_p(wa, wb, C::kQuant);
          if (C::kRowScale) {
            lw_sum = fmaf(wa, rinv[j].x, fmaf(wb, rinv[j].y, lw_sum));
          } else {
            l[hh] += p_lo(packed, C::kQuant) + p_hi(packed, C::kQuant);  // the weights the MMA uses
          }
          // rows 8j .. 8j+7 form 16-byte chunk j of the head's 128-byte row (128-byte swizzle)
          *reinterpret_cast<uint32_t*>(prow + ((j ^ (h & 7)) << 4)) = packed;
        }
        if (C::kRowScale && lw_sum > 0.f) l[hh] += lw_sum * fast_exp2(m_o[hh] - m_l[hh]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[sb]);
    }
    if (!dead) dead = !warp_wait(&ctl->o_done, 0, ctl, lane);
    float l_tot[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      l_tot[hh] = l[hh] + __shfl_xor_sync(kFull, l[hh], 1);
      l_tot[hh] += __shfl_xor_sync(kFull, l_tot[hh], 2);
    }
    if (p.cluster > 1) {
      // the cluster merges the splits (cluster_merge, below): publish this split's statistics
      if (c2 == 0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          ctl->st[hd[hh]] = dead ? make_float4(-INFINITY, -INFINITY, 0.f, 0.f)  // an empty split
                                 : make_float4(m_o[hh], m_l[hh], l_tot[hh], 0.f);
      }
    } else if (p.splits > 1) {
      if (!dead) {  // channel tiles 0-1; the loader warp of the same lane quarter writes 2-3
        tc_fence_after();
        store_partial(p, b, split, tmem, wq, lane, 0, kDim / 256);
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = hd[hh];
        if (c2 == 0 && h < p.heads) {
          float* ml = p.ml_part + ((size_t(b) * p.splits + split) * p.heads + h) * 4;
          *reinterpret_cast<float4*>(ml) = dead ? make_float4(-INFINITY, -INFINITY, 0.f, 0.f)  // empty partial
                                                : make_float4(m_o[hh], m_l[hh], l_tot[hh], 0.f);
        }
      }
    } else {
      // one split: normalise, inverse RoPE, store.  out = O * 2^(m_o - m_l) / l
      if (c2 == 0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          ctl->fin[hd[hh]] = (!dead && m_o[hh] != -INFINITY && l_tot[hh] > 0.f)
                                 ? fast_exp2(m_o[hh] - m_l[hh]) / l_tot[hh] : 0.f;
      }
      named_bar_sync();
      if (!dead) {
        tc_fence_after();
        const int r0 = kDim - p.rope_dim;
#pragma unroll 1
        for (int ct = 0; ct < kDim / 128; ++ct) {
          const int c = 128 * ct + 32 * wq + lane;
          const bool rot = c >= r0;
          const float cs = rot ? ctl->rope_cs[(c - r0) >> 1] : 1.f;
          const float sn = rot ? ctl->rope_sn[(c - r0) >> 1] : 0.f;
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + kColO + 64 * ct + 32 * half, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int hh = 32 * half + e;
              // (fin == 0: no rows, or a wait gave up; the accumulator was never written)
              float v = ctl->fin[hh] != 0.f ? __uint_as_float(o[e]) * ctl->fin[hh] : 0.f;
              const float partner = __shfl_xor_sync(kFull, v, 1);  // channel c ^ 1 of the same head
              if (rot) v = (c & 1) ? partner * sn + v * cs : v * cs - partner * sn;
              if (hh < p.heads) {
                const size_t oi = (size_t(b) * p.heads + hh) * kDim + c;
                if (p.out_fp32) static_cast<float*>(p.out)[oi] = v;
                else static_cast<uint16_t*>(p.out)[oi] = f2bf(v);
              }
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ loaders (warps 6..9)
    const int lw = warp - 6;
    // the CTA's selected indices, once, into shared memory
    // (a lane reads the index of its row straight from idx: one load per tile)
    if constexpr (C::kQuant) {
      // the first tile's loads go out before Q's conversion waits for Q
      QuantLoad<FMT> ql;
      if (nt > 0) ql.fetch(p, sq, b, t0, lw, lane);
      // Q: bf16 -> f16 in place (saturating), once per CTA
      if (warp_wait(&ctl->q_full, 0, ctl, lane)) {
        for (int v = threadIdx.x - 192; v < kQBytes / 16; v += 128) {
          uint4 x = *reinterpret_cast<const uint4*>(sQ + 16 * v);
          x = make_uint4(f32x2_to_f16x2_sat(bf16lo(x.x), bf16hi(x.x)), f32x2_to_f16x2_sat(bf16lo(x.y), bf16hi(x.y)),
                         f32x2_to_f16x2_sat(bf16lo(x.z), bf16hi(x.z)), f32x2_to_f16x2_sat(bf16lo(x.w), bf16hi(x.w)));
          *reinterpret_cast<uint4*>(sQ + 16 * v) = x;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->q_ready);
      }
      for (int i = 0; i < nt; ++i) {
        const int stage = i % kStages;
        if (i >= kStages && !warp_wait(&ctl->empty[stage], ((i / kStages) - 1) & 1, ctl, lane)) break;
        ql.put(ctl, stage, sR + stage * kTileBytes, lw, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->full[stage]);
        if (i + 1 < nt) ql.fetch(p, sq, b, t0 + i + 1, lw, lane);
      }
    } else {
      // rows: warp lw covers rows 16*lw .. 16*lw+15 of every tile
      for (int i = 0; i < nt; ++i) {
        const int T = t0 + i, stage = i % kStages;
        if (i >= kStages && !warp_wait(&ctl->empty[stage], ((i / kStages) - 1) & 1, ctl, lane)) break;
        uint8_t* tile = sR + stage * kTileBytes;
        if (!tile_tma(p, sq, b, T)) {
          // lane j < 16 resolves row 16*lw + j; every lane reads all 16 answers
          const RowSrc mine = row_source(p, sq, b, T, 16 * lw + (lane & 15));
          const uint32_t vb = __ballot_sync(kFull, mine.valid) & 0xffffu;
          if (lane == 0) ctl->vmask[stage][lw] = vb;
          // gathered bf16 rows: 16-byte cp.async into the 128-byte-swizzled tile
          // (rows that do not exist are zero-filled without a read)
          const uint8_t* base = static_cast<const uint8_t*>(mine.from_win ? p.win_codes : p.comp_codes);
#pragma unroll 4
          for (int j = 0; j < 16; ++j) {
            const int r = 16 * lw + j;
            const int64_t row = __shfl_sync(kFull, mine.row, j);
            const uint32_t bytes = (vb >> j) & 1u ? 16u : 0u;
            const uint8_t* src = base + size_t(row) * (kDim * 2);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int u_all = 32 * hh + lane;  // 16-byte unit of the 1 KB row
              const int c = u_all >> 3, u = u_all & 7;
              cp_async16_zfill(tile + c * kChunkBytes + r * 128 + ((u ^ (r & 7)) << 4), src + 16 * u_all, bytes);
            }
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
        }
        // (a TMA tile is brought by warp 0)
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->full[stage]);
      }
    }
    // the other half of the partial O^T (this warp's TMEM lane quarter is warp % 4)
    if (p.cluster == 1 && p.splits > 1 && warp_wait(&ctl->o_done, 0, ctl, lane)) {
      tc_fence_after();
      store_partial(p, b, split, tmem, warp & 3, lane, kDim / 256, kDim / 128);
    }
  }
  if (p.cluster > 1) cluster_merge(p, sq, ctl, reinterpret_cast<float*>(smem), tmem, b, split, warp, lane);
  // Retire: lane 0 of every warp arrives once the warp's own work is done
  // (in the TMA and MMA warps only lane 0 works), and warp 1 frees TMEM after
  // all ten arrivals.  A CTA-wide bar.sync here is not enough: its warps are
  // diverged (lanes 1-31 of warps 0 and 1 reach the end long before lane 0),
  // and such a barrier was seen to let warp 1 through before the epilogue
  // warps had finished reading TMEM.
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&ctl->retire);
  if (warp == 1) {
    if (lane == 0) retire_wait(&ctl->retire);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
    if (lane == 0 && ctl->abort) set_status(p.status, DSV4KV_DEV_TIMEOUT);
  }
}

// Merge split partials, normalise, inverse RoPE.  Per split: O_s (weights
// relative to 2^m_o), l_s (relative to 2^m_l):
//   out = [sum_s O_s 2^(m_o,s - Mo)] / [sum_s l_s 2^(m_l,s - Ml)] * 2^(Mo - Ml).
// One warp per (sequence, head), four per block.  Lane j owns channels
// 4j + 128q (q < 4) as float4s, so both channels of a rotary pair sit in one
// lane; lane s also owns split s's (m, l) terms, which the warp shares by
// shuffles.  The split loop's loads do not depend on each other.
constexpr int kCombWarps = 4;
constexpr int kCombFast = 4;  // splits up to which a warp issues all its loads at once

// The partial outputs are bf16 (half the bytes the decode CTAs write and the
// merges read); 4 channels of a split are one 8-byte load.
__device__ __forceinline__ float4 ld_bf16x4(const uint16_t* p) {
  const uint2 v = __ldcg(reinterpret_cast<const uint2*>(p));
  return make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
}

__global__ void __launch_bounds__(32 * kCombWarps) decode_combine(const uint16_t* __restrict__ o_part,
                                                                  const float* __restrict__ ml_part,
                                                                  const float* __restrict__ rope_tab, int splits,
                                                                  int heads, int bh_total, int rope_dim, int out_fp32,
                                                                  void* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x * kCombWarps + warp;
  if (bh >= bh_total) return;
  const int b = bh / heads, h = bh % heads;
  const size_t ml_stride = size_t(heads) * 4, o_stride = size_t(heads) * kDim;
  const float* mlb = ml_part + (size_t(b) * splits * heads + h) * 4;
  const uint16_t* ob = o_part + (size_t(b) * splits * heads + h) * kDim + 4 * lane;
  rope_tab += size_t(b) * kDim;  // this sequence's rotation
  // the rotation of this lane's rotary pairs (channels 128q + 4 lane + {0, 2}), read up front
  const int r0 = kDim - rope_dim;
  float cs[4][2], sn[4][2];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = 128 * q + 4 * lane + 2 * e;
      const bool rot = c >= r0;
      cs[q][e] = rot ? __ldcg(rope_tab + ((c - r0) >> 1)) : 1.f;
      sn[q][e] = rot ? __ldcg(rope_tab + kDim / 2 + ((c - r0) >> 1)) : 0.f;
    }
  float4 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  float mo = -INFINITY, ml = -INFINITY, L = 0.f;
  if (splits <= kCombFast) {
    // every load of the warp in one round trip: lane s holds split s's (m, l),
    // every lane its 16 channels of each split
    const float4 v = lane < splits ? __ldcg(reinterpret_cast<const float4*>(mlb + lane * ml_stride))
                                   : make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
    float4 x[kCombFast][4];
#pragma unroll
    for (int s = 0; s < kCombFast; ++s)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        x[s][q] = s < splits ? ld_bf16x4(ob + size_t(s) * o_stride + 128 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
    mo = v.x;
    ml = v.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mo = fmaxf(mo, __shfl_xor_sync(kFull, mo, o));
      ml = fmaxf(ml, __shfl_xor_sync(kFull, ml, o));
    }
    const float w = v.x == -INFINITY ? 0.f : exp2f(v.x - mo);
    L = v.y == -INFINITY ? 0.f : v.z * exp2f(v.y - ml);
#pragma unroll
    for (int s = 0; s < kCombFast; ++s) {
      const float ws = __shfl_sync(kFull, w, s);
      if (ws != 0.f) {  // an empty partial's O is never read (lanes >= splits carry w = 0)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q].x = fmaf(ws, x[s][q].x, acc[q].x);
          acc[q].y = fmaf(ws, x[s][q].y, acc[q].y);
          acc[q].z = fmaf(ws, x[s][q].z, acc[q].z);
          acc[q].w = fmaf(ws, x[s][q].w, acc[q].w);
        }
      }
    }
  } else {
    for (int s = lane; s < splits; s += 32) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(mlb + s * ml_stride));
      mo = fmaxf(mo, v.x);
      ml = fmaxf(ml, v.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mo = fmaxf(mo, __shfl_xor_sync(kFull, mo, o));
      ml = fmaxf(ml, __shfl_xor_sync(kFull, ml, o));
    }
    for (int s0 = 0; s0 < splits; s0 += 32) {
      float w = 0.f;
      if (s0 + lane < splits) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(mlb + (s0 + lane) * ml_stride));
        w = v.x == -INFINITY ? 0.f : exp2f(v.x - mo);
        if (v.y != -INFINITY) L += v.z * exp2f(v.y - ml);
      }
      const int cnt = min(32, splits - s0);
#pragma unroll 4
      for (int j = 0; j < cnt; ++j) {
        const float wj = __shfl_sync(kFull, w, j);
        const uint16_t* os = ob + size_t(s0 + j) * o_stride;
        float4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = ld_bf16x4(os + 128 * q);
        if (wj != 0.f) {  // an empty partial's O is never read
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[q].x = fmaf(wj, v[q].x, acc[q].x);
            acc[q].y = fmaf(wj, v[q].y, acc[q].y);
            acc[q].z = fmaf(wj, v[q].z, acc[q].z);
            acc[q].w = fmaf(wj, v[q].w, acc[q].w);
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(kFull, L, o);
  const float inv = (mo == -INFINITY || L <= 0.f) ? 0.f : exp2f(mo - ml) / L;
  const size_t ob_out = (size_t(b) * heads + h) * kDim;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = 128 * q + 4 * lane;
    float v[4] = {acc[q].x * inv, acc[q].y * inv, acc[q].z * inv, acc[q].w * inv};
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // identity rotation outside the rotary channels
      const float x = v[2 * e], y = v[2 * e + 1];
      v[2 * e] = x * cs[q][e] - y * sn[q][e];
      v[2 * e + 1] = x * sn[q][e] + y * cs[q][e];
    }
    if (out_fp32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + ob_out + c) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + ob_out + c) =
          make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    }
  }
}

// Merge for more than kCombFast splits.  Block (sequence, head, channel
// block cb) covers the CB-th part of the channels, [cb D/CB, (cb+1) D/CB):
// lane l of every warp owns channels cb D/CB + 128 q + 4l .. + 3 (float4s,
// q < 4/CB; both channels of a rotary pair sit in one float4), warp w the
// splits s = w mod kWideWarps, taken 2 CB at a time (one when CB = 1) with all their loads in
// flight before any is used.  Each warp keeps running maxima of the (m, l)
// terms it has seen, rescaling its sums when one grows (no separate pass
// over the maxima); the warps' sums, scaled to the block's maxima, meet in
// shared memory.  CB is chosen per launch so that the grid stays within a
// few blocks per SM.
constexpr int kWideWarps = 8;

template <int CB>
__global__ void __launch_bounds__(32 * kWideWarps, CB == 1 ? 4 : 2) decode_combine_wide(const uint16_t* __restrict__ o_part,
                                                                       const float* __restrict__ ml_part,
                                                                       const float* __restrict__ rope_tab, int splits,
                                                                       int heads, int rope_dim, int out_fp32,
                                                                       void* __restrict__ out) {
  constexpr int CW = kDim / CB;  // channels per block
  constexpr int Q = 4 / CB;      // float4s per lane and split
  constexpr int U = CB == 1 ? 1 : 2 * CB;  // splits per warp and round
  __shared__ __align__(16) float red[kWideWarps][CW];
  __shared__ float s_mo[kWideWarps], s_ml[kWideWarps], s_l[kWideWarps];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / CB, cb = blockIdx.x % CB;
  const int b = bh / heads, h = bh % heads;
  const size_t ml_stride = size_t(heads) * 4, o_stride = size_t(heads) * kDim;
  const float* mlb = ml_part + (size_t(b) * splits * heads + h) * 4;
  const uint16_t* ob = o_part + (size_t(b) * splits * heads + h) * kDim + CW * cb + 4 * lane;
  // this warp's splits, U per round, with running maxima (the warp's loads
  // are identical across its lanes, so every branch below is warp-uniform)
  float4 acc[Q];
#pragma unroll
  for (int q = 0; q < Q; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f, mo = -INFINITY, ml = -INFINITY;
  for (int s0 = warp; s0 < splits; s0 += kWideWarps * U) {
    float4 v[U], x[U][Q];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u * kWideWarps;
      v[u] = s < splits ? __ldcg(reinterpret_cast<const float4*>(mlb + s * ml_stride))
                        : make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u * kWideWarps;
#pragma unroll
      for (int q = 0; q < Q; ++q)
        x[u][q] = s < splits ? ld_bf16x4(ob + size_t(s) * o_stride + 128 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float rmo = mo, rml = ml;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      rmo = fmaxf(rmo, v[u].x);
      rml = fmaxf(rml, v[u].y);
    }
    if (rmo > mo) {  // rescale what the warp has summed so far to the new maximum
      const float a = mo == -INFINITY ? 0.f : exp2f(mo - rmo);
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        acc[q].x *= a;
        acc[q].y *= a;
        acc[q].z *= a;
        acc[q].w *= a;
      }
      mo = rmo;
    }
    if (rml > ml) {
      L *= ml == -INFINITY ? 0.f : exp2f(ml - rml);
      ml = rml;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (v[u].y != -INFINITY) L += v[u].z * exp2f(v[u].y - ml);
      if (v[u].x != -INFINITY) {  // an empty partial's O (m_o = -inf) is not used
        const float w = exp2f(v[u].x - mo);
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          acc[q].x = fmaf(w, x[u][q].x, acc[q].x);
          acc[q].y = fmaf(w, x[u][q].y, acc[q].y);
          acc[q].z = fmaf(w, x[u][q].z, acc[q].z);
          acc[q].w = fmaf(w, x[u][q].w, acc[q].w);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < Q; ++q) *reinterpret_cast<float4*>(&red[warp][128 * q + 4 * lane]) = acc[q];
  if (lane == 0) {  // every lane carries the same maxima and L
    s_mo[warp] = mo;
    s_ml[warp] = ml;
    s_l[warp] = L;
  }
  __syncthreads();
  if (threadIdx.x >= CW / 2) return;
  float mo_all = -INFINITY, ml_all = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWideWarps; ++w) {
    mo_all = fmaxf(mo_all, s_mo[w]);
    ml_all = fmaxf(ml_all, s_ml[w]);
  }
  float Lt = 0.f;
#pragma unroll
  for (int w = 0; w < kWideWarps; ++w)
    if (s_ml[w] != -INFINITY) Lt += s_l[w] * exp2f(s_ml[w] - ml_all);
  const float inv = (mo_all == -INFINITY || Lt <= 0.f) ? 0.f : exp2f(mo_all - ml_all) / Lt;
  const int cl = 2 * threadIdx.x, c = CW * cb + cl;  // CW/2 threads x 2 channels
  float v0 = 0.f, v1 = 0.f;
#pragma unroll
  for (int w = 0; w < kWideWarps; ++w) {
    if (s_mo[w] == -INFINITY) continue;  // a warp without a used partial
    const float a = exp2f(s_mo[w] - mo_all);
    const float2 x = *reinterpret_cast<const float2*>(&red[w][cl]);
    v0 = fmaf(a, x.x, v0);
    v1 = fmaf(a, x.y, v1);
  }
  v0 *= inv;
  v1 *= inv;
  const int r0 = kDim - rope_dim;
  if (c >= r0) {
    const int m = (c - r0) >> 1;
    const float* rt = rope_tab + size_t(b) * kDim;  // this sequence's rotation
    const float cs = __ldcg(rt + m), sn = __ldcg(rt + kDim / 2 + m);
    const float x = v0, y = v1;
    v0 = x * cs - y * sn;
    v1 = x * sn + y * cs;
  }
  const size_t o = (size_t(b) * heads + h) * kDim + c;
  if (out_fp32) *reinterpret_cast<float2*>(static_cast<float*>(out) + o) = make_float2(v0, v1);
  else static_cast<uint32_t*>(out)[o / 2] = pack_bf16x2(v0, v1);
}
static_assert(32 * kWideWarps >= kDim / 2, "enough threads to finish one channel pair each");

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
  uint16_t* o_part;
  float* ml_part;
  float* rope_tab;
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
  w.o_part = reinterpret_cast<uint16_t*>(take(sizeof(uint16_t) * size_t(batch) * pl.splits * heads * kDim));
  w.ml_part = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * pl.splits * heads * 4));
  w.rope_tab = reinterpret_cast<float*>(take(sizeof(float) * size_t(batch) * kDim));
  w.bytes = off;
  return w;
}

// Self-test of the bounded waits: one thread waits with wait_or_abort (as
// every wait of decode_kernel does) on an mbarrier that no thread arrives on,
// gives up after kWaitLimitNs, and flags DSV4KV_DEV_TIMEOUT.
__global__ void wait_timeout_probe(uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ Ctl ctl;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !wait_or_abort(&bar, 0, &ctl)) set_status(status, DSV4KV_DEV_TIMEOUT);
}

}  // namespace

dsv4kv_status selftest_wait_timeout_launch(uint32_t* status, cudaStream_t stream) {
  wait_timeout_probe<<<1, 32, 0, stream>>>(status);
  return check_launch("selftest_wait_timeout");
}

size_t decode_ws_bytes(int batch, int heads, int dim, int64_t rows_per_seq) {
  (void)dim;
  // rows_per_seq = compressed slots + window rows; the split plan only depends on the tile count
  const int tiles = int((rows_per_seq + kTileRows - 1) / kTileRows) + 1;
  Plan pl{};
  pl.splits = std::max(1, std::min(tiles, sm_count() / std::max(batch, 1)));  // upper bound of make_plan
  return decode_ws_layout(nullptr, batch, heads, pl).bytes;
}

// Shared-memory limit and cluster permission of decode_kernel<FMT>, once per device.
template <int FMT>
bool setup_fmt() {
  static std::atomic<uint64_t> attr_set{0};  // per instantiation, one bit per device
  if (done_on_device(attr_set)) return true;
  if (cudaFuncSetAttribute(decode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes)) !=
      cudaSuccess)
    return false;
  // clusters of 16 are beyond the portable size; without the permission the
  // occupancy query below answers 0 for them and they are not used
  cudaFuncSetAttribute(decode_kernel<FMT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaGetLastError();
  mark_done_on_device(attr_set);
  return true;
}

// How many clusters of C decode CTAs the device runs at once (0: none).
template <int FMT>
int active_clusters(int c) {
  static std::atomic<int> cache[5][64];  // [log2 C][device]; 0 = not queried, -1 = none
  int lc = 0;
  while ((1 << lc) < c) ++lc;
  std::atomic<int>& slot = cache[lc][current_device()];
  int n = slot.load(std::memory_order_relaxed);
  if (n == 0) {
    n = -1;
    if (setup_fmt<FMT>()) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(unsigned(c));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = unsigned(c);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int got = 0;
      if (cudaOccupancyMaxActiveClusters(&got, decode_kernel<FMT>, &cfg) == cudaSuccess && got > 0) n = got;
      cudaGetLastError();
    }
    slot.store(n, std::memory_order_relaxed);
  }
  return n > 0 ? n : 0;
}

template <int FMT>
dsv4kv_status launch_fmt(const CUtensorMap& tq, const CUtensorMap& tc, const CUtensorMap& tw, const Params& p,
                         int grid, cudaStream_t stream) {
  if (!setup_fmt<FMT>()) return check_launch("decode: cudaFuncSetAttribute");
  if (p.cluster > 1)
    launch_pdl_cluster(decode_kernel<FMT>, dim3(grid), dim3(kThreads), kSmemBytes, unsigned(p.cluster), stream, tq,
                       tc, tw, p);
  else
    launch_pdl(decode_kernel<FMT>, dim3(grid), dim3(kThreads), kSmemBytes, stream, tq, tc, tw, p);
  return check_launch("decode_kernel");
}

// The cluster size for a batch whose plan has s0 splits per sequence: the
// smallest power of two C >= s0 (C <= 16) whose clusters all run at once
// merges every sequence inside the kernel (no combine launch, splits = C);
// else the largest C that divides the split count rounded up to it, with one
// wave of clusters and at most one CTA per SM, merges groups of C splits; 1 = none.
// The environment variable DSV4KV_DECODE_MAX_CLUSTER (1, 2, 4, 8 or 16; read
// at every call) caps C.  The default is 1, the plain split-and-combine path:
// on B200, with the decode launched behind the selection kernel, the merge in
// clusters measured slower for every workload tried (c4a B=32 decode 26.9 us
// -> 32.7 us with C = 2, 34.4 us with C = 4; c128a B=1 t=2^20 17.4 -> 22.6 us),
// although it saves the combine launch and the partials' round trip.
template <int FMT>
void choose_cluster(int batch, int s0, int* cluster, int* splits) {
  *cluster = 1;
  *splits = s0;
  if (s0 <= 1) return;
  int cmax = 1;
  if (const char* e = std::getenv("DSV4KV_DECODE_MAX_CLUSTER")) {
    const int v = std::atoi(e);
    cmax = v >= 16 ? 16 : (v >= 8 ? 8 : (v >= 4 ? 4 : (v >= 2 ? 2 : 1)));
  }
  const int sms = sm_count();
  for (int c = 2; c <= cmax; c *= 2)
    if (c >= s0 && int64_t(batch) * c <= sms && active_clusters<FMT>(c) >= batch) {
      *cluster = c;
      *splits = c;
      return;
    }
  for (int c = cmax; c >= 2; c /= 2) {
    const int sp = (s0 + c - 1) / c * c;
    if (sp < 2 * c || int64_t(batch) * sp > sms) continue;
    if (int64_t(active_clusters<FMT>(c)) >= int64_t(batch) * (sp / c)) {
      *cluster = c;
      *splits = sp;
      return;
    }
  }
}

dsv4kv_status decode_launch(const DecodeArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (a.dim != kDim) return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: dim must be 512 (got %d)", a.dim);
  const int fmt = a.comp.fmt;
  if (a.win.fmt != fmt)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: the window cache must have the compressed cache's format");
  if (fmt != DSV4KV_BF16 && fmt != DSV4KV_FP8_E4M3_ROW && fmt != DSV4KV_FP4_E2M1_G16 &&
      fmt != DSV4KV_FP8_E4M3_ROW_ROPE_BF16)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: unknown cache format %d", fmt);
  if (fmt == DSV4KV_FP8_E4M3_ROW_ROPE_BF16 && a.rope_dim != 64)
    return set_error(DSV4KV_ERR_UNSUPPORTED, "decode: fp8 rows with bf16 rotary channels need rope_dim == 64");
  const int64_t slots = a.idx ? std::min<int64_t>(a.k, a.n) : a.n;
  const int comp_tiles = int((slots + kTileRows - 1) / kTileRows);
  const int win_tiles = (a.window + kTileRows - 1) / kTileRows;
  if (comp_tiles + win_tiles == 0) return set_error(DSV4KV_ERR_INVALID_ARG, "decode: no rows to attend");
  const Plan pl = make_plan(a.batch, comp_tiles, win_tiles);
  const DecodeWs w = decode_ws_layout(static_cast<char*>(ws), a.batch, a.heads, pl);
  if (ws_bytes < w.bytes) return set_error(DSV4KV_ERR_WORKSPACE, "decode: workspace too small");
  if (reinterpret_cast<uintptr_t>(ws) % 16 != 0)  // (the split statistics are 16-byte stores)
    return set_error(DSV4KV_ERR_INVALID_ARG, "decode: workspace not 16-byte aligned");

  CUtensorMap tq, tc, tw;
  // One box brings a whole operand in the layout the MMAs read: dimensions
  // (64 channels, rows, 8 channel chunks[, sequence]) land chunk-major, 64
  // rows x 128 bytes (128-byte swizzle) per chunk.
  {
    const uint64_t dims[4] = {64, uint64_t(a.heads), uint64_t(kChunks), uint64_t(a.batch)};
    const uint64_t strides[3] = {uint64_t(kDim) * 2, 128, uint64_t(a.heads) * kDim * 2};
    const uint32_t box[4] = {64, 64, uint32_t(kChunks), 1};
    if (!encode_tmap_nd(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the query tensor map");
  }
  const dsv4kv_cache& cc = a.comp;
  // rows a tensor map spans: the batch of dense caches, or a pool
  auto total_rows = [&](const dsv4kv_cache& c, const PageDesc& pg) -> uint64_t {
    const int64_t r = pg.table ? c.rows : int64_t(a.batch) * std::max<int64_t>(c.rows, 1);
    return std::max<uint64_t>(1, uint64_t(r));
  };
  if (fmt == DSV4KV_BF16) {
    // contiguous row runs: boxes of 64 channels x 64 rows, 128-byte swizzle
    auto rows_map = [&](CUtensorMap* m, const void* base, uint64_t rows) {
      const uint64_t dims[3] = {64, rows, uint64_t(kChunks)};
      const uint64_t strides[2] = {uint64_t(kDim) * 2, 128};
      const uint32_t box[3] = {64, uint32_t(kTileRows), uint32_t(kChunks)};
      return encode_tmap_nd(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    const void* comp_base = cc.codes ? cc.codes : a.win.codes;
    if (!rows_map(&tc, comp_base, total_rows(cc, a.comp_pg)))
      return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the compressed-cache tensor map");
    const void* win_base = a.win.codes ? a.win.codes : comp_base;
    if (!rows_map(&tw, win_base, total_rows(a.win, a.win_pg)))
      return set_error(DSV4KV_ERR_INVALID_ARG, "decode: cannot encode the window tensor map");
  } else {
    tc = tq;  // unused: quantised rows are loaded by the loader warps
    tw = tq;
  }

  Params p{};
  p.heads = a.heads;
  p.n = a.n;
  p.window = a.window;
  p.k = a.idx ? a.k : 0;
  int cluster = 1, splits = pl.splits;
  switch (fmt) {
    case DSV4KV_BF16: choose_cluster<DSV4KV_BF16>(a.batch, pl.splits, &cluster, &splits); break;
    case DSV4KV_FP8_E4M3_ROW: choose_cluster<DSV4KV_FP8_E4M3_ROW>(a.batch, pl.splits, &cluster, &splits); break;
    case DSV4KV_FP8_E4M3_ROW_ROPE_BF16:
      choose_cluster<DSV4KV_FP8_E4M3_ROW_ROPE_BF16>(a.batch, pl.splits, &cluster, &splits);
      break;
    default: choose_cluster<DSV4KV_FP4_E2M1_G16>(a.batch, pl.splits, &cluster, &splits); break;
  }
  p.splits = splits;
  p.cluster = cluster;
  p.t_seq = a.t_seq;
  p.t_max = a.t_max;
  p.stride = std::max(1, a.stride);
  p.comp_map = RowMap{a.comp_pg.table, std::max(1, a.comp_pg.page_rows), a.comp_pg.table_stride,
                      cc.rows, a.comp_pg.pool_pages};
  p.win_map = RowMap{a.win_pg.table, std::max(1, a.win_pg.page_rows), a.win_pg.table_stride, a.win.rows,
                     a.win_pg.pool_pages};
  p.idx = a.idx;
  p.comp_codes = static_cast<const uint8_t*>(cc.codes);
  p.comp_scales = cc.scales;
  p.win_codes = static_cast<const uint8_t*>(a.win.codes);
  p.win_scales = a.win.scales;
  p.score_scale = a.sm_scale * 1.4426950408889634f;
  p.o_part = w.o_part;
  p.ml_part = w.ml_part;
  p.rope_tab = w.rope_tab;
  p.status = w.status;
  p.t = a.t;
  p.rope_dim = a.rope_dim;
  p.rope_base = a.rope_base;
  p.out_fp32 = a.out_fp32;
  p.out = a.out;

  const int grid = a.batch * splits;
  dsv4kv_status st;
  switch (fmt) {
    case DSV4KV_BF16: st = launch_fmt<DSV4KV_BF16>(tq, tc, tw, p, grid, stream); break;
    case DSV4KV_FP8_E4M3_ROW: st = launch_fmt<DSV4KV_FP8_E4M3_ROW>(tq, tc, tw, p, grid, stream); break;
    case DSV4KV_FP8_E4M3_ROW_ROPE_BF16:
      st = launch_fmt<DSV4KV_FP8_E4M3_ROW_ROPE_BF16>(tq, tc, tw, p, grid, stream);
      break;
    default: st = launch_fmt<DSV4KV_FP4_E2M1_G16>(tq, tc, tw, p, grid, stream); break;
  }
  // one split, or one cluster per sequence: the decode kernel stored the output
  if (st != DSV4KV_OK || splits == 1 || cluster == splits) return st;
  const int parts = splits / cluster;  // partials per sequence left to merge
  const int bh_total = a.batch * a.heads;
  if (parts <= kCombFast)
    launch_pdl(decode_combine, dim3((bh_total + kCombWarps - 1) / kCombWarps), dim3(32 * kCombWarps), 0, stream,
               (const uint16_t*)w.o_part, (const float*)w.ml_part, (const float*)w.rope_tab, parts, a.heads,
               bh_total, a.rope_dim, a.out_fp32, a.out);
  else {
    // channel blocks per (sequence, head): as many as keep the grid within ~3 blocks per SM
    const int sms = sm_count();
    const int cb = bh_total * 4 <= 3 * sms ? 4 : (bh_total * 2 <= 3 * sms ? 2 : 1);
    auto kern = cb == 4 ? decode_combine_wide<4> : (cb == 2 ? decode_combine_wide<2> : decode_combine_wide<1>);
    launch_pdl(kern, dim3(bh_total * cb), dim3(32 * kWideWarps), 0, stream, (const uint16_t*)w.o_part,
               (const float*)w.ml_part, (const float*)w.rope_tab, parts, a.heads, a.rope_dim, a.out_fp32,
               a.out);
  }
  return check_launch("decode_combine");
}

}  // namespace dsv4kv
