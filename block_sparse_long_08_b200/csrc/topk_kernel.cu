// Top-k block choice over stored block scores (one warp per (b, g, t) row).
// See topk.cuh for the selection rule and its sources.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace msa {

namespace {

// Rows of up to 256 candidate blocks (query positions below 32,896 with
// 128-token blocks) take the threshold form with the row in registers;
// longer rows take the insertion scan.  (Four rows per warp with their
// networks interleaved measured slower: the extra registers cost more
// occupancy than the independent chains recovered.)
constexpr int kTopkVpl = 8;

__global__ void __launch_bounds__(256) msa_topk_kernel(const TopkArgs a) {
  __shared__ float s_cs[8][32];
  __shared__ int s_cj[8][32];
  const int w = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + w;
  const long long n_rows = (long long)a.B * a.G * a.L;
  if (row >= n_rows) return;
  const int t = (int)(row % a.L);
  const int bt = t / a.blk;
  if (bt <= 32 * kTopkVpl)
    warp_topk_select_thr<kTopkVpl>(a.scores + row * a.nb, bt, a.top_k, a.sel + row * a.top_k,
                                   s_cs[w], s_cj[w]);
  else
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
