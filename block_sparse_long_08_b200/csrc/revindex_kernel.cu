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
//   4. order   (when order_words > 0) each list sorted by query position,
//              so that the order -- and whatever is summed in it -- is the
//              same from run to run; pos_of follows.  A row selects a block
//              at most once, so the positions in a list are distinct.  Up
//              to kOrderCount entries: an entry's rank is the number of
//              smaller positions, counted in shared memory; up to
//              kOrderSort: a bitonic sort in shared memory; longer lists:
//              ranks read from a bitmap over the sequence's rows in the
//              chunk (and per-word prefix counts), the slot then found in
//              the row's selection.
// Every work item then holds <= qpi queries, so items cost the same and a
// persistent grid balances itself whatever the causal skew between early
// and late key blocks.
#include <cuda_runtime.h>

#include <climits>

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

constexpr int kOrderCount = 256;
constexpr int kOrderSort = 4096;
constexpr int kOrderThreads = 256;

// Exclusive prefix of x over the CTA's 256 threads; tot gets the sum (all
// threads).  warp_sums and total are shared scratch.
__device__ __forceinline__ int cta_exclusive_scan(int x, int *warp_sums, int *total, int &tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kOrderThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kOrderThreads / 32) warp_sums[lane] = w;
    if (lane == kOrderThreads / 32 - 1) *total = w;
  }
  __syncthreads();
  const int ex = v - x + (warp > 0 ? warp_sums[warp - 1] : 0);
  tot = *total;
  __syncthreads();   // warp_sums / total are rewritten by the next call
  return ex;
}

// Entry (t, slot) of list (b, g) now at list position pos: pos_of follows.
__device__ __forceinline__ void order_put(const RevIdxArgs &a, const int4 &s, int g, int x,
                                          int pos) {
  a.list[pos] = x;
  const int rl = s.x + ((x >> 5) - s.y) - a.r0;   // the row's index in the chunk
  a.pos_of[((long long)g * a.Rc + rl) * a.top_k + (x & 31)] = pos;
}

__global__ void __launch_bounds__(kOrderThreads) revidx_order_kernel(const RevIdxArgs a) {
  extern __shared__ int sm[];   // up to kOrderSort entries, or bitmap + prefix words
  __shared__ int warp_sums[32], total;
  const int n_lists = a.q.B * a.G * a.nb;
  const int tid = threadIdx.x;
  for (int bgj = blockIdx.x; bgj < n_lists; bgj += gridDim.x) {
    const int lo = a.list_off[bgj], n = a.list_off[bgj + 1] - lo;
    if (n <= 1) continue;   // the same for every thread of the CTA
    const int b = bgj / (a.G * a.nb), g = (bgj / a.nb) % a.G, j = bgj % a.nb;
    const int4 s = qgeo_seq(a.q, b);
    if (n <= kOrderCount) {
      for (int i = tid; i < n; i += kOrderThreads) sm[i] = a.list[lo + i];
      __syncthreads();
      for (int i = tid; i < n; i += kOrderThreads) {
        const int x = sm[i];
        int rank = 0;
        for (int m = 0; m < n; ++m) rank += sm[m] < x;
        order_put(a, s, g, x, lo + rank);
      }
      __syncthreads();
      continue;
    }
    if (n <= kOrderSort) {
      int np = kOrderCount;
      while (np < n) np <<= 1;
      for (int i = tid; i < np; i += kOrderThreads) sm[i] = i < n ? a.list[lo + i] : INT_MAX;
      __syncthreads();
      for (int k = 2; k <= np; k <<= 1) {   // ascending bitonic network over np entries
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
          for (int i = tid; i < np; i += kOrderThreads) {
            const int l = i ^ jj;
            if (l > i) {
              const int x = sm[i], y = sm[l];
              if ((x > y) == ((i & k) == 0)) {
                sm[i] = y;
                sm[l] = x;
              }
            }
          }
          __syncthreads();
        }
      }
      for (int i = tid; i < n; i += kOrderThreads) order_put(a, s, g, sm[i], lo + i);
      __syncthreads();
      continue;
    }
    // the sequence's rows in this chunk: positions [t_first, t_first + rows)
    const int r_first = max(a.r0, s.x);
    const int rows = min(a.r0 + a.Rc, s.x + s.z) - r_first;
    const int t_first = s.y + (r_first - s.x);
    const int nw = (rows + 31) >> 5;   // <= order_words (host bound)
    uint32_t *bits = reinterpret_cast<uint32_t *>(sm);
    int *pre = sm + a.order_words;
    for (int w = tid; w < nw; w += kOrderThreads) bits[w] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kOrderThreads) {
      const int u = (a.list[lo + i] >> 5) - t_first;
      atomicOr(&bits[u >> 5], 1u << (u & 31));
    }
    __syncthreads();
    int carry = 0;
    for (int base = 0; base < nw; base += kOrderThreads) {
      const int w = base + tid;
      const int c = w < nw ? __popc(bits[w]) : 0;
      int tile_total;
      const int ex = cta_exclusive_scan(c, warp_sums, &total, tile_total);
      if (w < nw) pre[w] = carry + ex;
      carry += tile_total;
    }
    __syncthreads();
    for (int w = tid; w < nw; w += kOrderThreads) {
      uint32_t m = bits[w];
      int pos = lo + pre[w];
      while (m) {
        const int bit = __ffs(m) - 1;
        m &= m - 1;
        const int t = t_first + w * 32 + bit;
        const long long srow =
            ((long long)s.w + (long long)g * a.q.sel_gs + (t - s.y)) * a.top_k;
        int slot = 0;
        for (int k = 0; k < a.top_k; ++k)
          if (a.sel[srow + k] == j) slot = k;
        order_put(a, s, g, t * 32 + slot, pos++);
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t revidx_order_smem(int order_words) {
  const size_t direct = sizeof(int) * kOrderSort;
  const size_t bitmap = sizeof(int) * 2 * size_t(order_words);
  return direct > bitmap ? direct : bitmap;
}

cudaError_t launch_revidx(const RevIdxArgs &a, cudaStream_t st) {
  const int n_cnt = a.q.B * a.G * a.nb;
  cudaError_t e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * n_cnt, st);
  if (e != cudaSuccess) return e;
  const long long n = (long long)a.G * a.Rc * a.top_k;
  const int grid = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  if (n > 0) revidx_count_kernel<<<grid, 256, 0, st>>>(a);
  revidx_scan_kernel<<<1, 1024, 0, st>>>(a);
  if (n > 0) revidx_fill_kernel<<<grid, 256, 0, st>>>(a);
  if (n > 0 && a.order_words > 0) {
    const size_t smem = revidx_order_smem(a.order_words);
    e = cudaFuncSetAttribute(revidx_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const int og = n_cnt < 148 * 8 ? n_cnt : 148 * 8;
    revidx_order_kernel<<<og, kOrderThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace msa
