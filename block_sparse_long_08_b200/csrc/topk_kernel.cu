// Top-k block choice over stored block scores (one warp per (b, g, t) row).
// See topk.cuh for the selection rule and its sources.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace msa {

namespace {

__global__ void __launch_bounds__(256) msa_topk_kernel(const TopkArgs a) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long n_rows = (long long)a.B * a.G * a.L;
  if (row >= n_rows) return;
  const int t = (int)(row % a.L);
  const int bt = t / kBlock;
  warp_topk_select(a.scores + row * a.nb, bt, a.top_k, a.sel + row * a.top_k);
}

}  // namespace

cudaError_t launch_topk_kernel(const TopkArgs &a, cudaStream_t st) {
  const long long n_rows = (long long)a.B * a.G * a.L;
  if (n_rows == 0) return cudaSuccess;
  const long long grid = (n_rows + 7) / 8;
  msa_topk_kernel<<<(unsigned)grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
