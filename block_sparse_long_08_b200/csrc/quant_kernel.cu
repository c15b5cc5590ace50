// Row-wise quantization of bf16 rows to the OCP FP8 E4M3 format with one
// fp32 scale per row, the storage of an FP8 index-key cache (the long-context
// essay's low-precision cache direction).  scale = max|x| / 448 (448 being
// the largest finite E4M3 magnitude; 1 for an all-zero row) and code = E4M3
// round-to-nearest-even of x / scale, saturated.  One warp per row.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace msa {

namespace {

// Two fp32 values -> two E4M3 codes (lo in the low byte), RNE, saturated.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(256) quantize_e4m3_rows_kernel(const uint16_t *__restrict__ x,
                                                                 long long rows, int cols,
                                                                 uint8_t *__restrict__ codes,
                                                                 float *__restrict__ scale) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint16_t *xr = x + row * cols;
  float amax = 0.f;
  for (int c = lane * 8; c < cols; c += 256) {
    const uint4 v = *reinterpret_cast<const uint4 *>(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (lane == 0) scale[row] = s;
  uint8_t *cr = codes + row * cols;
  for (int c = lane * 8; c < cols; c += 256) {
    const uint4 v = *reinterpret_cast<const uint4 *>(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t two = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[i]), s), __fdiv_rn(bf16_hi(w[i]), s));
      packed[i >> 1] |= two << (16 * (i & 1));
    }
    *reinterpret_cast<uint2 *>(cr + c) = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3_rows(const uint16_t *x, long long rows, int cols, uint8_t *codes,
                                      float *scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const long long grid = (rows + 7) / 8;
  quantize_e4m3_rows_kernel<<<(unsigned)grid, 256, 0, st>>>(x, rows, cols, codes, scale);
  return cudaGetLastError();
}

}  // namespace msa
