// GPU twin of the seeded input generator in datagen/__init__.py: the same
// SplitMix64 counter recipe, the same Irwin-Hall(12) normal and multiply-shift
// uniform integers, so host and device produce bit-identical input bytes.
// Input generation only: none of the method's arithmetic lives here.
#include <cstdint>
#include <cuda_runtime.h>

#define DG_API extern "C" __attribute__((visibility("default")))

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}
__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ull); }

__device__ __forceinline__ uint16_t normal_bf16(uint64_t key, uint64_t e) {
  int64_t total = 0;
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const uint64_t d = draw(key, 3 * e + j);
    total += int64_t(d & 0xffff) + int64_t((d >> 16) & 0xffff) + int64_t((d >> 32) & 0xffff) + int64_t(d >> 48);
  }
  const float f = float(total - 393210) * (1.0f / 65536.0f);  // exact: <= 19 significant bits
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

__device__ __forceinline__ int64_t uniform_int(uint64_t key, uint64_t e, int64_t lo, int64_t hi) {
  const uint64_t d = draw(key, e);
  const uint64_t span = uint64_t(hi - lo + 1);
  return lo + int64_t(((d >> 32) * span) >> 32);
}

__global__ void k_normal_bf16(uint16_t* out, uint64_t key, uint64_t offset, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    out[i] = normal_bf16(key, offset + uint64_t(i));
}

__global__ void k_int_bf16(uint16_t* out, uint64_t key, uint64_t offset, int64_t n, int64_t lo, int64_t hi) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float f = float(uniform_int(key, offset + uint64_t(i), lo, hi));
    out[i] = uint16_t(__float_as_uint(f) >> 16);  // small integers are exact in bf16
  }
}

// fp4 indexer keys of `rows` rows x di channels, rows starting at row0:
// v = U{0..13}: nibble = (v / 7) << 3 | (v % 7); every scale byte 0x40.
__global__ void k_fp4_keys(uint8_t* codes, uint8_t* scales, uint64_t key, uint64_t row0, int64_t rows, int di) {
  const int64_t nbytes = rows * (di / 2);
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < nbytes; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / (di / 2);
    const int cb = int(i % (di / 2));
    const uint64_t e0 = (row0 + uint64_t(r)) * uint64_t(di) + uint64_t(2 * cb);
    const int64_t v0 = uniform_int(key, e0, 0, 13), v1 = uniform_int(key, e0 + 1, 0, 13);
    const uint32_t n0 = uint32_t(((v0 / 7) << 3) | (v0 % 7)), n1 = uint32_t(((v1 / 7) << 3) | (v1 % 7));
    codes[i] = uint8_t(n0 | (n1 << 4));
    if (cb < di / 16) scales[r * (di / 16) + cb] = 0x40;
  }
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  return int(g < 148 * 32 ? (g < 1 ? 1 : g) : 148 * 32);
}

}  // namespace

DG_API int dg_normal_bf16(void* out, uint64_t key, uint64_t offset, int64_t n, void* stream) {
  if (n <= 0) return 0;
  k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, key, offset, n);
  return int(cudaGetLastError());
}

DG_API int dg_int_bf16(void* out, uint64_t key, uint64_t offset, int64_t n, int64_t lo, int64_t hi, void* stream) {
  if (n <= 0) return 0;
  k_int_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, key, offset, n, lo, hi);
  return int(cudaGetLastError());
}

DG_API int dg_fp4_index_keys(void* codes, void* scales, uint64_t key, uint64_t row0, int64_t rows, int di, void* stream) {
  if (rows <= 0) return 0;
  k_fp4_keys<<<grid_for(rows * (di / 2)), 256, 0, (cudaStream_t)stream>>>((uint8_t*)codes, (uint8_t*)scales, key, row0,
                                                                         rows, di);
  return int(cudaGetLastError());
}
