// Warp-level top-k block choice with the forced local block.
//
// researchpapers.dev "MiniMax Sparse Attention", section "机制": keep the
// top-k blocks per (query, group) and always keep the most recent local
// block; section "2048 个 KV token": top_k counts every kept block, so
// top_k - 1 come from the earlier blocks.  Equal scores go to the lower
// block id.
//
// A warp keeps the best k1 = top_k-1 (score, id) pairs in (score desc, id
// asc) order, one pair per lane, and a threshold (the worst kept score).
// Candidates are offered 32 at a time, in increasing id order; only lanes
// beating the threshold enter a ballot, and those are inserted one at a time
// in lane order with shuffles.  Because candidates arrive in id order, an
// equal score never displaces a kept entry, which is the lower-id rule.  For
// unstructured scores the expected number of insertions over n blocks is
// about k*ln(n/k), so a pass costs about one coalesced read of the row.  The
// kept ids plus the local block are finally sorted ascending by a 32-lane
// bitonic network.
#pragma once
#include <cfloat>
#include <climits>
#include <cstdint>

namespace msa {

struct WarpTopk {
  float ls;   // this lane's kept score (lane < k1)
  int lj;     // this lane's kept id
  float thr;  // worst kept score (warp-uniform)
};

__device__ __forceinline__ void warp_topk_init(WarpTopk &st) {
  st.ls = -FLT_MAX;
  st.lj = INT_MAX;
  st.thr = -FLT_MAX;
}

// (score desc, id asc) order: true if (sa, ja) ranks ahead of (sb, jb).
__device__ __forceinline__ bool ranks_ahead(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

// First offer into an empty list: sort the 32 candidates with a bitonic
// network in (score desc, id asc) order and keep the first k1, instead of
// inserting them one at a time.
__device__ __forceinline__ void warp_topk_seed(WarpTopk &st, float s, int j, bool valid, int k1) {
  const int lane = threadIdx.x & 31;
  float ks = valid ? s : -FLT_MAX;
  int kj = valid ? j : INT_MAX;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int d = k >> 1; d > 0; d >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, ks, d);
      const int oj = __shfl_xor_sync(0xffffffffu, kj, d);
      const bool first = (lane & k) == 0;   // this k-block is ordered best-first
      const bool lower = (lane & d) == 0;
      const bool mine_ahead = ranks_ahead(ks, kj, os, oj);
      const bool keep = (lower == first) ? mine_ahead : !mine_ahead;
      ks = keep ? ks : os;
      kj = keep ? kj : oj;
    }
  }
  st.ls = (lane < k1) ? ks : -FLT_MAX;
  st.lj = (lane < k1) ? kj : INT_MAX;
  st.thr = __shfl_sync(0xffffffffu, st.ls, k1 - 1);
}

// Offer one candidate per lane (s, j, valid); lanes' candidates must be in
// increasing id order across lanes and after every earlier offer.
__device__ __forceinline__ void warp_topk_offer(WarpTopk &st, float s, int j, bool valid, int k1) {
  const int lane = threadIdx.x & 31;
  unsigned m = __ballot_sync(0xffffffffu, valid && (s > st.thr));
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    const float cs = __shfl_sync(0xffffffffu, s, src);
    const int cj = __shfl_sync(0xffffffffu, j, src);
    if (cs > st.thr) {
      const int p = __popc(__ballot_sync(0xffffffffu, lane < k1 && st.ls >= cs));
      const float us = __shfl_up_sync(0xffffffffu, st.ls, 1);
      const int uj = __shfl_up_sync(0xffffffffu, st.lj, 1);
      if (lane < k1 && lane > p) { st.ls = us; st.lj = uj; }
      if (lane == p) { st.ls = cs; st.lj = cj; }
      st.thr = __shfl_sync(0xffffffffu, st.ls, k1 - 1);
    }
  }
}

// Offer the scores of blocks [lo, hi) of `row`, four coalesced loads ahead.
__device__ __forceinline__ void warp_topk_scan(WarpTopk &st, const float *__restrict__ row, int lo,
                                               int hi, int k1) {
  const int lane = threadIdx.x & 31;
  for (int base = lo; base < hi; base += 128) {
    float s4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + u * 32 + lane;
      s4[u] = (j < hi) ? __ldg(row + j) : -FLT_MAX;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int jb = base + u * 32;
      if (jb >= hi) break;
      const bool empty = __all_sync(0xffffffffu, st.lj == INT_MAX);  // warp-uniform
      if (empty)
        warp_topk_seed(st, s4[u], jb + lane, jb + lane < hi, k1);
      else
        warp_topk_offer(st, s4[u], jb + lane, jb + lane < hi, k1);
    }
  }
}

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

// Kept ids + local block bt, ascending, into out[0..top_k).
__device__ __forceinline__ void warp_topk_write(const WarpTopk &st, int bt, int top_k,
                                                int32_t *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int k1 = top_k - 1;
  int id = (lane < k1) ? st.lj : (lane == k1 ? bt : INT_MAX);
  id = warp_bitonic_sort_asc(id, lane);
  if (lane < top_k) out[lane] = id;
}

// Descending bitonic sort of one float per lane (lane 0 ends with the
// largest).
__device__ __forceinline__ float warp_sort_desc(float x, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, x, j);
      const bool first = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      x = (lower == first) ? fmaxf(x, o) : fminf(x, o);
    }
  }
  return x;
}

// Threshold form of the same selection, for rows of at most 32 * VPL
// scores (held in registers).  Lane l holds scores l, l+32, ...; T, the
// k1-th largest of the 32 lane maxima, has at least k1 scores at or above
// it (those lane maxima), so the k1-th score of the row is >= T and every
// kept block scores >= T.  The few candidates >= T (about 20 for k1 = 15 on
// unstructured scores) are gathered in id order through shared memory and
// ranked once with the bitonic (score desc, id asc) network; more than 32
// candidates (exact ties, adversarial rows) fall back to the insertion
// scan.  Same result as warp_topk_select, ties included.
// s_cs / s_cj: 32 floats / ints of shared memory per warp.
template <int VPL>
__device__ __forceinline__ void warp_topk_select_thr(const float *__restrict__ row, int bt,
                                                     int top_k, int32_t *__restrict__ out,
                                                     float *s_cs, int *s_cj) {
  const int lane = threadIdx.x & 31;
  if (bt + 1 <= top_k) {
    for (int k = lane; k < top_k; k += 32) out[k] = (k <= bt) ? k : -1;
    return;
  }
  if (top_k == 1) {
    if (lane == 0) out[0] = bt;
    return;
  }
  const int k1 = top_k - 1;
  float v[VPL];
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {   // every load issued before any use
    const int j = i * 32 + lane;
    v[i] = (j < bt) ? __ldg(row + j) : -FLT_MAX;
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) m = fmaxf(m, v[i]);
  const float T = __shfl_sync(0xffffffffu, warp_sort_desc(m, lane), k1 - 1);
  int c = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) c += (i * 32 + lane < bt && v[i] >= T) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  WarpTopk st;
  if (total <= 32) {
    int pos = incl - c;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (i * 32 + lane < bt && v[i] >= T) {
        s_cs[pos] = v[i];
        s_cj[pos] = i * 32 + lane;
        ++pos;
      }
    }
    __syncwarp();
    const bool have = lane < total;
    const float cs = have ? s_cs[lane] : -FLT_MAX;
    const int cj = have ? s_cj[lane] : INT_MAX;
    __syncwarp();   // the next row of this warp rewrites the exchange area
    warp_topk_seed(st, cs, cj, have, k1);
  } else {
    warp_topk_init(st);
    warp_topk_scan(st, row, 0, bt, k1);
  }
  warp_topk_write(st, bt, top_k, out);
}

// The selection rule for the block-score row of a query whose local block
// is bt: blocks 0..bt-1 are candidates (the local block is not read).
// Writes top_k ints to out: selected ids ascending, -1 padding.
__device__ __forceinline__ void warp_topk_select(const float *__restrict__ row, int bt, int top_k,
                                                 int32_t *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  if (bt + 1 <= top_k) {
    for (int k = lane; k < top_k; k += 32) out[k] = (k <= bt) ? k : -1;
    return;
  }
  if (top_k == 1) {            // only the local block
    if (lane == 0) out[0] = bt;
    return;
  }
  WarpTopk st;
  warp_topk_init(st);
  warp_topk_scan(st, row, 0, bt, top_k - 1);
  warp_topk_write(st, bt, top_k, out);
}

}  // namespace msa
