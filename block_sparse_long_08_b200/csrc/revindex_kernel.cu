// Reverse index of a block selection ("query gathering" / "reverse index"
// of researchpapers.dev "MiniMax Sparse Attention", section "对工程团队的意义";
// "KV external aggregation Q" of the baguaai.com 稀疏注意力 MSA entry).
//
// For a query chunk [t0, t0+Lc) it lists, for every (b, g, key block j),
// the (query, slot) pairs whose selection holds j -- a counting sort of the
// selection by key block:
//   1. count   cnt[b,g,j] += 1 for every selected entry
//   2. scan    list_off = exclusive scan of cnt,
//              item_off = exclusive scan of ceil(cnt / qpi)  (work items of
//              at most qpi queries, i.e. 128 query-head rows, per block)
//   3. fill    list[list_off[bgj] + k] = t * 32 + slot  (order inside a
//              list is arbitrary: each (t, slot) partial is computed
//              independently of the others in its tile)
// Every work item then holds <= qpi queries, so items cost the same and a
// persistent grid balances itself whatever the causal skew between early
// and late key blocks.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace msa {

namespace {

__global__ void __launch_bounds__(256) revidx_count_kernel(const RevIdxArgs a) {
  const long long n = (long long)a.B * a.G * a.Lc * a.top_k;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(e % a.top_k);
    const long long r = e / a.top_k;
    const int tl = (int)(r % a.Lc);
    const long long bg = r / a.Lc;
    const int j = a.sel[(bg * a.L + a.t0 + tl) * a.top_k + k];
    if (j < 0) continue;
    if (j >= a.nb) {
      atomicCAS(a.status, 0, kStatusBadInput);
      continue;
    }
    atomicAdd(&a.cnt[bg * a.nb + j], 1);
  }
}

// Single CTA, 1024 threads: exclusive scans of cnt and ceil(cnt/qpi).
__global__ void __launch_bounds__(1024) revidx_scan_kernel(const RevIdxArgs a) {
  __shared__ int warp_a[32], warp_b[32];
  const int n = a.B * a.G * a.nb;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per;
  const int hi = min(n, lo + per);
  int sa = 0, sb = 0;
  for (int x = lo; x < hi; ++x) {
    const int c = a.cnt[x];
    sa += c;
    sb += (c + a.qpi - 1) / a.qpi;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = sa, ib = sb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o);
    const int yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += ya; ib += yb; }
  }
  if (lane == 31) { warp_a[warp] = ia; warp_b[warp] = ib; }
  __syncthreads();
  if (warp == 0) {
    int va = warp_a[lane], vb = warp_b[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, va, o);
      const int yb = __shfl_up_sync(0xffffffffu, vb, o);
      if (lane >= o) { va += ya; vb += yb; }
    }
    warp_a[lane] = va;
    warp_b[lane] = vb;
  }
  __syncthreads();
  int ea = ia - sa + (warp > 0 ? warp_a[warp - 1] : 0);
  int eb = ib - sb + (warp > 0 ? warp_b[warp - 1] : 0);
  for (int x = lo; x < hi; ++x) {
    const int c = a.cnt[x];
    a.list_off[x] = ea;
    a.item_off[x] = eb;
    a.cursor[x] = 0;
    ea += c;
    eb += (c + a.qpi - 1) / a.qpi;
  }
  if (threadIdx.x == blockDim.x - 1) {
    a.list_off[n] = warp_a[31];
    a.item_off[n] = warp_b[31];
  }
}

__global__ void __launch_bounds__(256) revidx_fill_kernel(const RevIdxArgs a) {
  const long long n = (long long)a.B * a.G * a.Lc * a.top_k;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(e % a.top_k);
    const long long r = e / a.top_k;
    const int tl = (int)(r % a.Lc);
    const long long bg = r / a.Lc;
    const int t = a.t0 + tl;
    const int j = a.sel[(bg * a.L + t) * a.top_k + k];
    if (j < 0 || j >= a.nb) continue;
    const long long bgj = bg * a.nb + j;
    const int pos = a.list_off[bgj] + atomicAdd(&a.cursor[bgj], 1);
    a.list[pos] = t * 32 + k;
  }
}

}  // namespace

cudaError_t launch_revidx(const RevIdxArgs &a, cudaStream_t st) {
  const int n_cnt = a.B * a.G * a.nb;
  cudaError_t e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * n_cnt, st);
  if (e != cudaSuccess) return e;
  const long long n = (long long)a.B * a.G * a.Lc * a.top_k;
  const int grid = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  revidx_count_kernel<<<grid, 256, 0, st>>>(a);
  revidx_scan_kernel<<<1, 1024, 0, st>>>(a);
  revidx_fill_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
