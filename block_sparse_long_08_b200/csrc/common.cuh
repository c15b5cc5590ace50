// Shared constants and small device helpers of the MSA kernels.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace msa {

// Device status word values (mirror MSA_ERR_* in msa.h).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -5;
constexpr int kStatusBadInput = -6;

constexpr int kBlock = 128;   // KV block length
constexpr int kHeadDim = 128; // d
constexpr int kMaxTopK = 32;

// Workspace header: status word + scratch counters.
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace msa
