// Cache quantiser: fp8 E4M3 with one fp32 scale per row, or fp4 E2M1 with one
// E4M3 scale per 16 channels.
//
// [P1] quantisation paragraphs: the attention cache uses fp8 ("partly
// token-wise fp8") and the indexer cache fp4; [P3] "storing the main KV in
// FP4": E2M1 values with one E4M3 scale per 16 channels.  Arithmetic (fixed
// here because the pages give no rounding rule):
//   fp8 row:  scale = fp32(amax / 448) (1 when amax == 0);
//             code = E4M3_rn_satfinite(fp32(x / scale)).
//   fp4 group of 16: s = E4M3_rn_satfinite(fp32(amax / 6));
//             code = E2M1_rn_satfinite(fp32(x / value(s))), 0 when value(s) == 0.
//   fp8 with bf16 rotary channels ([P1]: the RoPE dimensions stay in bf16):
//             the fp8 row rule over the first D - 64 channels (amax over
//             those only), then the last 64 channels as bf16 (nearest even);
//             a row is D - 64 code bytes followed by the 64 bf16 values.
// Divisions are IEEE round-to-nearest: by a row's (or group's) scale s they
// use Markstein's method (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/s), q0 = RN(x y), the remainder r = x - s q0 is exact in one FMA
// and RN(q0 + r y) = RN(x / s), which holds while nothing under- or
// overflows: the quotients here are at most 448 in magnitude, scales outside
// [2^-64, 2^64] take __fdiv_rn instead (so y is a normal number), and
// quotients small enough for r to underflow round to a zero code either way.
// The sign of a zero quotient is restored after the correction.  Conversions use the hardware
// cvt.rn.satfinite instructions.  One warp per row.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace dsv4kv {

namespace {

constexpr int kRowsPerBlock = 8;

__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;  // lo in bits 0..7, hi in bits 8..15
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r & 0xffu;  // lo in bits 0..3, hi in bits 4..7
}
// x / s rounded to nearest for every x of a row or group that shares s.
struct RnDivider {
  float s, y;  // the divisor and RN(1 / s)
  bool fast;
  __device__ __forceinline__ float operator()(float x) const {
    if (!fast) return __fdiv_rn(x, s);
    const float q0 = x * y;
    const float r = fmaf(-q0, s, x);
    // The correction turns a quotient of -0 into +0; the sign of x / s is
    // the sign of q0 (s > 0), so it is put back.
    return copysignf(fmaf(r, y, q0), q0);
  }
};
__device__ __forceinline__ RnDivider rn_divider(float s) {
  RnDivider d;
  d.s = s;
  d.y = __frcp_rn(s);
  d.fast = s >= 0x1p-64f && s <= 0x1p64f;  // false for NaN
  return d;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const float v = __uint_as_float((c & 0x7fu) << 20) * 0x1p120f;
  return (c & 0x80u) ? -v : v;
}

template <int PER, bool IN_FP32, int FMT>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
    quantize_kernel(const void* __restrict__ in, int64_t rows, uint8_t* __restrict__ codes, void* __restrict__ scales) {
  constexpr int D = 32 * PER;
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;
  float x[PER];
  if (IN_FP32) {
    const float* src = static_cast<const float*>(in) + size_t(row) * D + PER * lane;
#pragma unroll
    for (int v = 0; v < PER / 4; ++v) {
      const float4 f = *reinterpret_cast<const float4*>(src + 4 * v);
      x[4 * v] = f.x;
      x[4 * v + 1] = f.y;
      x[4 * v + 2] = f.z;
      x[4 * v + 3] = f.w;
    }
  } else {
    const uint16_t* src = static_cast<const uint16_t*>(in) + size_t(row) * D + PER * lane;
#pragma unroll
    for (int v = 0; v < PER / 4; ++v) {
      const uint2 u = *reinterpret_cast<const uint2*>(src + 4 * v);
      x[4 * v] = bf16lo(u.x);
      x[4 * v + 1] = bf16hi(u.x);
      x[4 * v + 2] = bf16lo(u.y);
      x[4 * v + 3] = bf16hi(u.y);
    }
  }
  if (FMT == DSV4KV_FP8_E4M3_ROW_ROPE_BF16) {
    // lanes [0, BL) hold the fp8 body, lanes [BL, 32) the 64 rotary channels
    constexpr int BL = 32 - 64 / PER;
    const bool body = lane < BL;
    float amax = 0.f;
    if (body) {
#pragma unroll
      for (int e = 0; e < PER; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const RnDivider div = rn_divider(scale);
    uint8_t* row_dst = codes + size_t(row) * (D + 64);
    if (body) {
      uint32_t packed[PER / 4];
#pragma unroll
      for (int v = 0; v < PER / 4; ++v) {
        const uint32_t lo = cvt_e4m3x2(div(x[4 * v + 1]), div(x[4 * v]));
        const uint32_t hi = cvt_e4m3x2(div(x[4 * v + 3]), div(x[4 * v + 2]));
        packed[v] = lo | (hi << 16);
      }
#pragma unroll
      for (int v = 0; v < PER / 4; ++v) reinterpret_cast<uint32_t*>(row_dst + PER * lane)[v] = packed[v];
    } else {
      // bf16 of fp32 input rounds to nearest even; bf16 input is reproduced exactly
      uint32_t* dst = reinterpret_cast<uint32_t*>(row_dst + (D - 64) + 2 * PER * (lane - BL));
#pragma unroll
      for (int v = 0; v < PER / 2; ++v) dst[v] = pack_bf16x2(x[2 * v], x[2 * v + 1]);
    }
    if (lane == 0) static_cast<float*>(scales)[row] = scale;
  } else if (FMT == DSV4KV_FP8_E4M3_ROW) {
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const RnDivider div = rn_divider(scale);
    uint32_t packed[PER / 4];
#pragma unroll
    for (int v = 0; v < PER / 4; ++v) {
      const uint32_t lo = cvt_e4m3x2(div(x[4 * v + 1]), div(x[4 * v]));
      const uint32_t hi = cvt_e4m3x2(div(x[4 * v + 3]), div(x[4 * v + 2]));
      packed[v] = lo | (hi << 16);
    }
    uint8_t* dst = codes + size_t(row) * D + PER * lane;
#pragma unroll
    for (int v = 0; v < PER / 4; ++v) reinterpret_cast<uint32_t*>(dst)[v] = packed[v];
    if (lane == 0) static_cast<float*>(scales)[row] = scale;
  } else {
    // groups of 16 channels: inside a lane (PER >= 16) or across 16/PER lanes
    constexpr int G = PER >= 16 ? 16 : PER;        // channels of a group held by this lane
    constexpr int NG = PER / G;                    // groups (or group parts) per lane
    constexpr int LANES_PER_GROUP = 16 / G;
    float s_val[NG];
    uint32_t s_code[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < G; ++e) amax = fmaxf(amax, fabsf(x[G * g + e]));
#pragma unroll
      for (int o = 1; o < LANES_PER_GROUP; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      s_code[g] = cvt_e4m3x2(0.f, __fdiv_rn(amax, 6.f)) & 0xffu;
      s_val[g] = e4m3_value(s_code[g]);
    }
    RnDivider divs[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) divs[g] = rn_divider(s_val[g] > 0.f ? s_val[g] : 1.f);
    uint8_t* dst = codes + size_t(row) * (D / 2) + (PER / 2) * lane;
    uint32_t packed[PER / 8 > 0 ? PER / 8 : 1];
#pragma unroll
    for (int v = 0; v < (PER + 7) / 8; ++v) packed[v] = 0;
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const float s = s_val[e / G];
      const RnDivider& div = divs[e / G];
      const uint32_t byte = s > 0.f ? cvt_e2m1x2(div(x[e + 1]), div(x[e])) : 0u;
      packed[e / 8] |= byte << (8 * ((e / 2) & 3));
    }
    if (PER >= 8) {
#pragma unroll
      for (int v = 0; v < PER / 8; ++v) reinterpret_cast<uint32_t*>(dst)[v] = packed[v];
    } else {
#pragma unroll
      for (int e = 0; e < PER / 2; ++e) dst[e] = uint8_t(packed[0] >> (8 * e));
    }
    uint8_t* sdst = static_cast<uint8_t*>(scales) + size_t(row) * (D / 16);
    if (PER >= 16) {
#pragma unroll
      for (int g = 0; g < NG; ++g) sdst[NG * lane + g] = uint8_t(s_code[g]);
    } else if (lane % LANES_PER_GROUP == 0) {
      sdst[lane / LANES_PER_GROUP] = uint8_t(s_code[0]);
    }
  }
}

template <int PER>
dsv4kv_status launch_per(const void* in, int in_fp32, int64_t rows, int fmt, void* codes, void* scales,
                         cudaStream_t stream) {
  const dim3 grid(unsigned((rows + kRowsPerBlock - 1) / kRowsPerBlock));
  const dim3 block(32 * kRowsPerBlock);
  uint8_t* c = static_cast<uint8_t*>(codes);
  if (fmt == DSV4KV_FP8_E4M3_ROW) {
    if (in_fp32) quantize_kernel<PER, true, DSV4KV_FP8_E4M3_ROW><<<grid, block, 0, stream>>>(in, rows, c, scales);
    else quantize_kernel<PER, false, DSV4KV_FP8_E4M3_ROW><<<grid, block, 0, stream>>>(in, rows, c, scales);
  } else if (fmt == DSV4KV_FP8_E4M3_ROW_ROPE_BF16) {
    if (in_fp32)
      quantize_kernel<PER, true, DSV4KV_FP8_E4M3_ROW_ROPE_BF16><<<grid, block, 0, stream>>>(in, rows, c, scales);
    else
      quantize_kernel<PER, false, DSV4KV_FP8_E4M3_ROW_ROPE_BF16><<<grid, block, 0, stream>>>(in, rows, c, scales);
  } else {
    if (in_fp32) quantize_kernel<PER, true, DSV4KV_FP4_E2M1_G16><<<grid, block, 0, stream>>>(in, rows, c, scales);
    else quantize_kernel<PER, false, DSV4KV_FP4_E2M1_G16><<<grid, block, 0, stream>>>(in, rows, c, scales);
  }
  return check_launch("quantize_kernel");
}

}  // namespace

dsv4kv_status quantize_launch(const void* in, int in_fp32, int64_t rows, int dim, int fmt, void* codes,
                              void* scales, cudaStream_t stream) {
  if (rows == 0) return DSV4KV_OK;
  switch (dim) {
    case 128: return launch_per<4>(in, in_fp32, rows, fmt, codes, scales, stream);
    case 256: return launch_per<8>(in, in_fp32, rows, fmt, codes, scales, stream);
    case 512: return launch_per<16>(in, in_fp32, rows, fmt, codes, scales, stream);
    case 1024: return launch_per<32>(in, in_fp32, rows, fmt, codes, scales, stream);
    default: return set_error(DSV4KV_ERR_UNSUPPORTED, "quantize: dim must be 128, 256, 512 or 1024 (got %d)", dim);
  }
}

}  // namespace dsv4kv
