// Reverse index of a block selection ("query gathering" / "reverse index"
// of researchpapers.dev "MiniMax Sparse Attention", section "对工程团队的意义";
// "KV external aggregation Q" of the baguaai.com 稀疏注意力 MSA entry).
//
// For a query chunk (the packed query rows [r0, r0+Rc), see QGeo) it lists,
// for every (b, g, key block j), the (query, slot) pairs whose selection
// holds j -- a counting sort of the selection by key block:
//   1. count   cnt[b,g,j] += 1 for every selected entry; the value before
//              the increment (the entry's rank among the entries of block
//              j) is kept in pos_of
//   2. scan    list_off = exclusive scan of cnt,
//              item_off = exclusive scan of ceil(cnt / qpi)  (work items of
//              at most qpi queries, i.e. 128 query-head rows, per block)
//   3. fill    pos = list_off[bgj] + rank; list[pos] = t * 32 + slot and
//              pos_of[g, row, slot] = pos (the inverse map by which the
//              merge finds a row's partials).  No atomics: the order inside
//              a list is whatever order the count's atomics produced, and
//              each (t, slot) partial is computed independently of the
//              others in its tile.
// Every work item then holds <= qpi queries, so items cost the same and a
// persistent grid balances itself whatever the causal skew between early
// and late key blocks.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace msa {

namespace {

// Entry e of the chunk, in [G][Rc][top_k] order: its group, sequence,
// position and selection slot address.
struct RevEntry {
  int k, g, b, t;
  long long sel_idx;
};
__device__ __forceinline__ RevEntry rev_entry(const RevIdxArgs &a, long long e) {
  RevEntry x;
  x.k = (int)(e % a.top_k);
  const long long gr = e / a.top_k;
  const int rl = (int)(gr % a.Rc);
  x.g = (int)(gr / a.Rc);
  const int r = a.r0 + rl;
  x.b = qgeo_seq_of_row(a.q, r);
  const int4 s = qgeo_seq(a.q, x.b);
  x.t = s.y + (r - s.x);
  x.sel_idx = ((long long)s.w + (long long)x.g * a.q.sel_gs + (r - s.x)) * a.top_k + x.k;
  return x;
}

__global__ void __launch_bounds__(256) revidx_count_kernel(const RevIdxArgs a) {
  const long long n = (long long)a.G * a.Rc * a.top_k;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const RevEntry x = rev_entry(a, e);
    const int j = a.sel[x.sel_idx];
    if (j < 0) continue;
    if (j >= a.nb) {
      atomicCAS(a.status, 0, kStatusBadInput);
      continue;
    }
    a.pos_of[e] = atomicAdd(&a.cnt[((long long)x.b * a.G + x.g) * a.nb + j], 1);
  }
}

// Block-wide inclusive scan of (x, y) pairs over 1024 threads; returns the
// pair totals through *tot (shared).
__device__ __forceinline__ void block_scan2(int &x, int &y, int *warp_x, int *warp_y, int *tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yx = __shfl_up_sync(0xffffffffu, x, o);
    const int yy = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) { x += yx; y += yy; }
  }
  if (lane == 31) { warp_x[warp] = x; warp_y[warp] = y; }
  __syncthreads();
  if (warp == 0) {
    int vx = warp_x[lane], vy = warp_y[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yx = __shfl_up_sync(0xffffffffu, vx, o);
      const int yy = __shfl_up_sync(0xffffffffu, vy, o);
      if (lane >= o) { vx += yx; vy += yy; }
    }
    warp_x[lane] = vx;
    warp_y[lane] = vy;
    if (lane == 31) { tot[0] = vx; tot[1] = vy; }
  }
  __syncthreads();
  if (warp > 0) { x += warp_x[warp - 1]; y += warp_y[warp - 1]; }
}

// Single CTA, 1024 threads: exclusive scans of cnt and ceil(cnt/qpi), in
// tiles of 4096 entries (4 consecutive entries per thread, 16-byte loads).
__global__ void __launch_bounds__(1024) revidx_scan_kernel(const RevIdxArgs a) {
  __shared__ int warp_x[32], warp_y[32], tot[2];
  const int n = a.q.B * a.G * a.nb;
  int carry_x = 0, carry_y = 0;
  for (int base = 0; base < n; base += 4096) {
    const int i0 = base + 4 * threadIdx.x;
    int c[4];
    if (i0 + 3 < n) {
      const int4 v = *reinterpret_cast<const int4 *>(a.cnt + i0);
      c[0] = v.x; c[1] = v.y; c[2] = v.z; c[3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) c[u] = (i0 + u < n) ? a.cnt[i0 + u] : 0;
    }
    int ch[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ch[u] = (c[u] + a.qpi - 1) / a.qpi;
    const int sx = c[0] + c[1] + c[2] + c[3];
    const int sy = ch[0] + ch[1] + ch[2] + ch[3];
    int x = sx, y = sy;
    block_scan2(x, y, warp_x, warp_y, tot);
    int ex = carry_x + x - sx, ey = carry_y + y - sy;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i0 + u < n) {
        a.list_off[i0 + u] = ex;
        a.item_off[i0 + u] = ey;
      }
      ex += c[u];
      ey += ch[u];
    }
    carry_x += tot[0];
    carry_y += tot[1];
    __syncthreads();   // tot / warp sums are rewritten by the next tile
  }
  if (threadIdx.x == 0) {
    a.list_off[n] = carry_x;
    a.item_off[n] = carry_y;
  }
}

__global__ void __launch_bounds__(256) revidx_fill_kernel(const RevIdxArgs a) {
  const long long n = (long long)a.G * a.Rc * a.top_k;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const RevEntry x = rev_entry(a, e);
    const int j = a.sel[x.sel_idx];
    if (j < 0 || j >= a.nb) continue;
    const int pos = a.list_off[((long long)x.b * a.G + x.g) * a.nb + j] + a.pos_of[e];
    a.list[pos] = x.t * 32 + x.k;
    a.pos_of[e] = pos;
  }
}

}  // namespace

cudaError_t launch_revidx(const RevIdxArgs &a, cudaStream_t st) {
  const int n_cnt = a.q.B * a.G * a.nb;
  cudaError_t e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * n_cnt, st);
  if (e != cudaSuccess) return e;
  const long long n = (long long)a.G * a.Rc * a.top_k;
  const int grid = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  if (n > 0) revidx_count_kernel<<<grid, 256, 0, st>>>(a);
  revidx_scan_kernel<<<1, 1024, 0, st>>>(a);
  if (n > 0) revidx_fill_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
