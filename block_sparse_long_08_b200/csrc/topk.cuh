// Warp-level top-k block choice with the forced local block.
//
// researchpapers.dev "MiniMax Sparse Attention", section "机制": keep the
// top-k blocks per (query, group) and always keep the most recent local
// block; section "2048 个 KV token": top_k counts every kept block, so
// top_k - 1 come from the earlier blocks.  Equal scores go to the lower
// block id.
//
// One warp handles one row of block scores.  The warp keeps the best
// top_k-1 (score, id) pairs sorted in descending order, one pair per lane,
// and a threshold (the worst kept score).  Scores are read 32 at a time,
// coalesced; only lanes beating the threshold enter a ballot, and those
// candidates are inserted one at a time in lane order (ascending id) with
// shuffles.  For unstructured scores the expected number of insertions over
// n blocks is about k*ln(n/k), so the pass costs about one coalesced read of
// the row.  The kept ids plus the local block are then sorted ascending by
// a 32-lane bitonic network.
#pragma once
#include <cfloat>
#include <climits>
#include <cstdint>

namespace msa {

__device__ __forceinline__ int warp_bitonic_sort_asc(int v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool up = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      v = (lower == up) ? min(v, o) : max(v, o);
    }
  }
  return v;
}

// row: scores of blocks 0..bt-1 (the local block bt is not read).
// Writes top_k ints to out: selected ids ascending, -1 padding.
__device__ __forceinline__ void warp_topk_select(const float *__restrict__ row, int bt, int top_k,
                                                 int32_t *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  if (bt + 1 <= top_k) {
    for (int k = lane; k < top_k; k += 32) out[k] = (k <= bt) ? k : -1;
    return;
  }
  const int k1 = top_k - 1;
  float ls = -FLT_MAX;
  int lj = INT_MAX;
  float thr = -FLT_MAX;
  for (int base = 0; base < bt; base += 128) {
    float s4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + u * 32 + lane;
      s4[u] = (j < bt) ? __ldg(row + j) : -FLT_MAX;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int jb = base + u * 32;
      if (jb >= bt) break;
      const float s = s4[u];
      unsigned m = __ballot_sync(0xffffffffu, (jb + lane < bt) && (s > thr));
      while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1;
        const float cs = __shfl_sync(0xffffffffu, s, src);
        if (cs > thr) {
          const int p = __popc(__ballot_sync(0xffffffffu, lane < k1 && ls >= cs));
          const float us = __shfl_up_sync(0xffffffffu, ls, 1);
          const int uj = __shfl_up_sync(0xffffffffu, lj, 1);
          if (lane < k1 && lane > p) { ls = us; lj = uj; }
          if (lane == p) { ls = cs; lj = jb + src; }
          thr = __shfl_sync(0xffffffffu, ls, k1 - 1);
        }
      }
    }
  }
  int id = (lane < k1) ? lj : (lane == k1 ? bt : INT_MAX);
  id = warp_bitonic_sort_asc(id, lane);
  if (lane < top_k) out[lane] = id;
}

}  // namespace msa
