// Decode step ("MiniMax M3 sparse attention" explainer, mlqm.cn/news/533796,
// §4.1: the new token scores the whole cache with the index branch and then
// attends only to its selected blocks, which cuts KV bandwidth by about an
// order of magnitude).  Everything here is bound by HBM bandwidth; the
// dominant stream is the k_idx cache scan (seq_len * d_idx * 2 bytes per
// sequence).
//
//   decode_index_kernel   one warp per (sequence, 128-key chunk before the
//                         local block): scores of the keys against all G
//                         index queries with mma.sync m16n8k16 (N = 8
//                         groups), then the per-group block max (one block
//                         per chunk, or two with 64-token blocks).  k_idx
//                         rows stream straight from HBM in 16-byte loads.
//   decode_topk_kernel    one CTA per (sequence, group): 16 warps scan
//                         segments of the block scores, one warp merges.
//   decode_attn_kernel    split over selected blocks: one CTA per
//                         (sequence, group, slot) computes the block's
//                         partial softmax for the R heads of the group on
//                         the tensor cores (mma.sync, heads as M rows); the
//                         last CTA of each (sequence, group) to finish, found
//                         with an atomic ticket, merges the <= top_k
//                         partials into the output.
// The top-k and attention kernels are launched as programmatic dependents
// of the kernel before them (their launch overlaps its tail) and wait for
// its results with griddepcontrol.wait before reading them.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace msa {

namespace {

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Programmatic dependent launch: wait until the grid this kernel depends on
// has completed and its memory is visible (a no-op without the launch
// attribute).
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Called by every CTA of decode_attn_kernel once its partial (or, for an
// unused slot, its -inf lse) is written.  The last of the top_k CTAs of
// (sequence b, group g) to get here merges the slot partials of the group's
// R heads: o = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M), M = max lse_s.
// Warp w takes heads w, w+4, ...: lane s holds lse_s, and each lane merges
// four columns, with the slots' loads issued 16 at a time before any sum
// (this merge ends the decode step, so its latency is on the critical
// path).  The ticket counters are zeroed by decode_topk_kernel.
template <int R>
__device__ __forceinline__ void dec_merge_if_last(const DecodeArgs &a, int b, int g) {
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __threadfence();   // this CTA's partial, visible before its ticket
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.tickets[b * a.G + g], 1) == a.top_k - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int hh = warp; hh < R; hh += 4) {
    const size_t p0 = (size_t(b) * a.H + size_t(g) * R + hh) * a.top_k;
    const float my = lane < a.top_k ? __ldcg(a.part_lse + p0 + lane) : -INFINITY;
    float M = my;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float wm = (my > -INFINITY) ? __expf(my - M) : 0.f;
    float wsum = wm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < a.top_k; s0 += 16) {
      float4 v[16];
#pragma unroll
      for (int s = 0; s < 16; ++s)
        v[s] = (s0 + s < a.top_k)
                   ? __ldcg(reinterpret_cast<const float4 *>(a.part_o + (p0 + s0 + s) * kHeadDim) + lane)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const float w = __shfl_sync(0xffffffffu, wm, (s0 + s) & 31);
        if (s0 + s < a.top_k && w > 0.f) {
          acc.x = fmaf(w, v[s].x, acc.x);
          acc.y = fmaf(w, v[s].y, acc.y);
          acc.z = fmaf(w, v[s].z, acc.z);
          acc.w = fmaf(w, v[s].w, acc.w);
        }
      }
    }
    const float inv = (M > -INFINITY && wsum > 0.f) ? 1.f / wsum : 0.f;
    uint2 r;
    r.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    r.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(a.out + (size_t(b) * a.H + size_t(g) * R + hh) * kHeadDim +
                               lane * 4) = r;
  }
}

// Reduce a warp's per-lane block maxima over the 8 lanes of each group pair
// and store them: block jb0 of groups 2c, 2c+1 (lanes c < 4), and with
// 64-token blocks also block jb0 + 1 unless it is the local block bt.
template <int BLK>
__device__ __forceinline__ void store_block_max(const DecodeArgs &a, int b, int jb0, int bt,
                                                int lane, float mx0, float mx1, float my0,
                                                float my1) {
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    if (BLK == 64) {
      my0 = fmaxf(my0, __shfl_xor_sync(0xffffffffu, my0, o));
      my1 = fmaxf(my1, __shfl_xor_sync(0xffffffffu, my1, o));
    }
  }
  if (lane < 4) {
    const int g0 = 2 * lane, g1 = 2 * lane + 1;
    float *s0 = a.scores + (size_t(b) * a.G + g0) * a.nb_max;
    float *s1 = a.scores + (size_t(b) * a.G + g1) * a.nb_max;
    if (g0 < a.G) s0[jb0] = mx0;
    if (g1 < a.G) s1[jb0] = mx1;
    if (BLK == 64 && jb0 + 1 < bt) {
      if (g0 < a.G) s0[jb0 + 1] = my0;
      if (g1 < a.G) s1[jb0 + 1] = my1;
    }
  }
}

// A warp scores one 128-key chunk against the (up to 8) index queries of
// its sequence.  The MMA's k dimension is a fixed permutation of d_idx
// applied to both operands, chosen so that each lane reads whole 16-byte
// granules of k_idx: for k-step kk = 2m + h, lane (g4 = lane/4, c = lane%4)
// feeds d = 8(c + 4m) + 4h + {0,1} at k positions 2c, 2c+1 and
// d = 8(c + 4m) + 4h + {2,3} at k positions 2c+8, 2c+9.
template <int DI, int BLK>
__global__ void __launch_bounds__(256) decode_index_kernel(const DecodeArgs a) {
  constexpr int NM = DI / 32;  // 16-byte granules per lane per key row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = blockIdx.x * 8 + warp;   // 128-key chunk
  const int n = a.seq_lens[b];
  if (n < 1 || n > a.Lmax) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(a.status, 0, kStatusBadInput);
    return;
  }
  const int bt = (n - 1) / BLK;          // local block
  const int jb0 = (BLK == 128) ? j : 2 * j;   // first block of the chunk
  if (bt + 1 <= a.top_k || jb0 >= bt) return;
  // with 64-token blocks, the chunk's second half may be the local block
  const int nrt = (BLK == 128 || jb0 + 1 < bt) ? 8 : 4;   // 16-key row tiles to score
  const int g4 = lane >> 2, c = lane & 3;
  // B fragments: q_idx[b, group g4, permuted d]
  uint32_t bf[NM][2][2];
  {
    const bool gv = g4 < a.G;
    const uint16_t *qrow = a.q_idx + (size_t(b) * a.G + (gv ? g4 : 0)) * DI;
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 v = *reinterpret_cast<const uint2 *>(qrow + 8 * (c + 4 * m) + 4 * h);
        bf[m][h][0] = gv ? v.x : 0u;
        bf[m][h][1] = gv ? v.y : 0u;
      }
  }
  const uint16_t *kbase = a.k_idx_cache + (size_t(b) * a.Lmax + size_t(j) * 128) * DI;
  float mx0 = -FLT_MAX, mx1 = -FLT_MAX;   // first block of the chunk, groups 2c, 2c+1
  float my0 = -FLT_MAX, my1 = -FLT_MAX;   // second block (BLK 64)
#pragma unroll 2
  for (int rt = 0; rt < nrt; ++rt) {
    const uint16_t *r0 = kbase + size_t(rt * 16 + g4) * DI;
    const uint16_t *r1 = r0 + 8 * DI;
    uint4 lo[NM], hi[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      lo[m] = ldg_nc_v4(r0 + 8 * (c + 4 * m));
      hi[m] = ldg_nc_v4(r1 + 8 * (c + 4 * m));
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      mma_bf16_16816(acc, lo[m].x, hi[m].x, lo[m].y, hi[m].y, bf[m][0][0], bf[m][0][1]);
      mma_bf16_16816(acc, lo[m].z, hi[m].z, lo[m].w, hi[m].w, bf[m][1][0], bf[m][1][1]);
    }
    if (BLK == 128 || rt < 4) {
      mx0 = fmaxf(mx0, fmaxf(acc[0], acc[2]));
      mx1 = fmaxf(mx1, fmaxf(acc[1], acc[3]));
    } else {
      my0 = fmaxf(my0, fmaxf(acc[0], acc[2]));
      my1 = fmaxf(my1, fmaxf(acc[1], acc[3]));
    }
  }
  store_block_max<BLK>(a, b, jb0, bt, lane, mx0, mx1, my0, my1);
}

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte first) -> two f16 (exact: every E4M3 value is an
// f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  const uint16_t in = static_cast<uint16_t>(two);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
  return r;
}

__device__ __forceinline__ uint32_t f16x2_of(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// decode_index_kernel for an FP8 index-key cache: the stored key of token s
// is k_idx_scale[s] * E4M3(k_idx8[s]) (one scale per token), so its score is
// k_idx_scale[s] * (q_idx . E4M3 codes).  Half the bytes of the bf16 scan.
// The MMA runs in f16: the codes convert exactly, and q_idx (bf16) converts
// exactly while it stays within the f16 range.  Lane (g4, c) loads 16-byte
// granules of 16 codes; k-step kk takes d = 16(c + 4(kk/4)) + 4(kk%4) +
// {0,1} at k positions 2c, 2c+1 and + {2,3} at 2c+8, 2c+9, i.e. the bytes
// of word kk%4 of granule kk/4.
template <int DI, int BLK>
__global__ void __launch_bounds__(256) decode_index_fp8_kernel(const DecodeArgs a) {
  constexpr int NG = DI / 64;  // granules per lane per key row
  constexpr int NK = DI / 16;  // MMA k-steps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = blockIdx.x * 8 + warp;   // 128-key chunk
  const int n = a.seq_lens[b];
  if (n < 1 || n > a.Lmax) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(a.status, 0, kStatusBadInput);
    return;
  }
  const int bt = (n - 1) / BLK;
  const int jb0 = (BLK == 128) ? j : 2 * j;
  if (bt + 1 <= a.top_k || jb0 >= bt) return;
  const int nrt = (BLK == 128 || jb0 + 1 < bt) ? 8 : 4;
  const int g4 = lane >> 2, c = lane & 3;
  uint32_t bq[NK][2];
  {
    const bool gv = g4 < a.G;
    const uint16_t *qrow = a.q_idx + (size_t(b) * a.G + (gv ? g4 : 0)) * DI;
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
      const int d0 = 16 * (c + 4 * (kk >> 2)) + 4 * (kk & 3);
      const uint2 v = *reinterpret_cast<const uint2 *>(qrow + d0);
      bq[kk][0] = gv ? f16x2_of(bf16_lo(v.x), bf16_hi(v.x)) : 0u;
      bq[kk][1] = gv ? f16x2_of(bf16_lo(v.y), bf16_hi(v.y)) : 0u;
    }
  }
  const uint8_t *kbase = a.k_idx8 + (size_t(b) * a.Lmax + size_t(j) * 128) * DI;
  const float *sbase = a.k_idx_scale + size_t(b) * a.Lmax + size_t(j) * 128;
  float mx0 = -FLT_MAX, mx1 = -FLT_MAX, my0 = -FLT_MAX, my1 = -FLT_MAX;
#pragma unroll 2
  for (int rt = 0; rt < nrt; ++rt) {
    const uint8_t *r0 = kbase + size_t(rt * 16 + g4) * DI;
    const uint8_t *r1 = r0 + 8 * DI;
    uint4 lo[NG], hi[NG];
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      lo[gi] = ldg_nc_v4(r0 + 16 * (c + 4 * gi));
      hi[gi] = ldg_nc_v4(r1 + 16 * (c + 4 * gi));
    }
    const float s0 = __ldg(sbase + rt * 16 + g4), s1 = __ldg(sbase + rt * 16 + g4 + 8);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      const uint32_t wl[4] = {lo[gi].x, lo[gi].y, lo[gi].z, lo[gi].w};
      const uint32_t wh[4] = {hi[gi].x, hi[gi].y, hi[gi].z, hi[gi].w};
#pragma unroll
      for (int w = 0; w < 4; ++w)
        mma_f16_16816(acc, e4m3x2_to_f16x2(wl[w]), e4m3x2_to_f16x2(wh[w]),
                      e4m3x2_to_f16x2(wl[w] >> 16), e4m3x2_to_f16x2(wh[w] >> 16),
                      bq[4 * gi + w][0], bq[4 * gi + w][1]);
    }
    if (BLK == 128 || rt < 4) {
      mx0 = fmaxf(mx0, fmaxf(acc[0] * s0, acc[2] * s1));
      mx1 = fmaxf(mx1, fmaxf(acc[1] * s0, acc[3] * s1));
    } else {
      my0 = fmaxf(my0, fmaxf(acc[0] * s0, acc[2] * s1));
      my1 = fmaxf(my1, fmaxf(acc[1] * s0, acc[3] * s1));
    }
  }
  store_block_max<BLK>(a, b, jb0, bt, lane, mx0, mx1, my0, my1);
}

// One CTA per (sequence, group): 16 warps each keep the top_k-1 of a
// contiguous segment of the block scores, then warp 0 merges the 16 lists
// (segment by segment, each in (score desc, id asc) order, so an equal
// score always arrives after the lower id it ties with).
constexpr int kTopkWarps = 16;

__global__ void __launch_bounds__(kTopkWarps * 32) decode_topk_kernel(const DecodeArgs a) {
  __shared__ float cand_s[kTopkWarps][32];
  __shared__ int cand_j[kTopkWarps][32];
  const int row = blockIdx.x;  // b * G + g
  const int b = row / a.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();                              // the scan's block scores
  if (threadIdx.x == 0) a.tickets[row] = 0;    // the attention's merge ticket
  const int n = a.seq_lens[b];
  int32_t *out = a.sel + size_t(row) * a.top_k;
  if (n < 1 || n > a.Lmax) {
    if (warp == 0 && lane < a.top_k) out[lane] = -1;
    return;
  }
  const int bt = (n - 1) / a.blk;
  if (bt + 1 <= a.top_k) {
    if (warp == 0)
      for (int k = lane; k < a.top_k; k += 32) out[k] = (k <= bt) ? k : -1;
    return;
  }
  if (a.top_k == 1) {            // only the local block
    if (threadIdx.x == 0) out[0] = bt;
    return;
  }
  const int k1 = a.top_k - 1;
  const int seg = ((bt + kTopkWarps * 32 - 1) / (kTopkWarps * 32)) * 32;
  const int lo = warp * seg, hi = min(bt, lo + seg);
  WarpTopk st;
  warp_topk_init(st);
  if (lo < hi) warp_topk_scan(st, a.scores + size_t(row) * a.nb_max, lo, hi, k1);
  cand_s[warp][lane] = st.ls;
  cand_j[warp][lane] = st.lj;
  __syncthreads();
  if (warp == 0) {
    // Every warp's k1-th score bounds the final k1-th score from below, so
    // only candidates at or above the largest of them can survive.
    float t0 = -FLT_MAX;
    for (int w = 0; w < kTopkWarps; ++w)
      if (cand_j[w][k1 - 1] != INT_MAX) t0 = fmaxf(t0, cand_s[w][k1 - 1]);
    WarpTopk m;
    warp_topk_init(m);
    for (int w = 0; w < kTopkWarps; ++w) {
      const int cj = cand_j[w][lane];
      const float cs = cand_s[w][lane];
      const bool ok = lane < k1 && cj != INT_MAX && cs >= t0;
      if (w == 0)
        warp_topk_seed(m, cs, cj, ok, k1);
      else
        warp_topk_offer(m, cs, cj, ok, k1);
    }
    warp_topk_write(m, bt, a.top_k, out);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// One CTA (4 warps) per (slot, group, sequence) computes the block's partial
// softmax for the R <= 16 heads of the group on the tensor cores
// (mma.sync m16n8k16, heads as the 16 M rows):
//   S = q K^T: warp w owns keys 32w..32w+31 (four 8-key n-tiles).  K rows are
//     the B operand, read straight from HBM as 16-byte granules with the same
//     d permutation as the decode index scan (applied to q as well).
//   softmax: row max / sum with shuffles over the lanes of a row and shared
//     memory across the 4 warps; keys past the query are masked.
//   O = P V: S's accumulator fragments are exactly P's A fragments (two
//     8-key n-tiles form one 16-key k-step); V is staged in shared memory
//     (rows padded to 272 B) and read with ldmatrix.trans.  The 4 warps'
//     partial O are summed through shared memory.
constexpr int kVPitch = kHeadDim + 8;  // bf16 per staged V row (272 B: conflict-free ldmatrix)
template <int R, int BLK>
constexpr int dec_attn_area() {
  // staged V; the 4 warps' partial O reuse the area once every warp has
  // read V (with 128-token blocks the V rows are the larger of the two)
  return (BLK * kVPitch * 2 > 4 * R * kHeadDim * 4) ? BLK * kVPitch * 2 : 4 * R * kHeadDim * 4;
}
template <int R, int BLK>
constexpr int dec_attn_smem() {
  // the V / partial-O area, then the row max / sum exchange (6 CTAs fit on
  // an SM with 128-token blocks)
  return dec_attn_area<R, BLK>() + 2 * 4 * 16 * 4;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <int R, int BLK>
__global__ void __launch_bounds__(128) decode_attn_kernel(const DecodeArgs a) {
  constexpr int KW = BLK / 4;   // keys per warp
  constexpr int NT = KW / 8;    // 8-key n-tiles per warp
  extern __shared__ __align__(16) uint8_t dsm[];
  uint16_t *sV = reinterpret_cast<uint16_t *>(dsm);
  float *s_o = reinterpret_cast<float *>(dsm);                     // [4 warps][R rows][128], over V
  float *s_m = reinterpret_cast<float *>(dsm + dec_attn_area<R, BLK>());   // [4][16]
  float *s_l = s_m + 4 * 16;                                        // [4][16]
  const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, c = lane & 3;
  griddep_wait();   // the top-k's selection
  const int n = a.seq_lens[b];
  const int j = (n >= 1 && n <= a.Lmax) ? a.sel[(size_t(b) * a.G + g) * a.top_k + slot] : -1;
  const size_t prow0 = (size_t(b) * a.H + size_t(g) * R) * a.top_k + slot;
  if (j < 0) {   // an unused slot: an empty partial
    if (tid < R) a.part_lse[prow0 + size_t(tid) * a.top_k] = -INFINITY;
    dec_merge_if_last<R>(a, b, g);
    return;
  }
  const int t = n - 1;
  const int nvis = min(BLK, t - j * BLK + 1);
  const size_t row_stride = size_t(a.G) * kHeadDim;
  const uint16_t *kb = a.k_cache + ((size_t(b) * a.Lmax + size_t(j) * BLK) * a.G + g) * kHeadDim;
  const uint16_t *vb = a.v_cache + ((size_t(b) * a.Lmax + size_t(j) * BLK) * a.G + g) * kHeadDim;
  // V block -> shared memory (coalesced 16-byte cp.async), overlapping S
  const uint32_t sV_u = static_cast<uint32_t>(__cvta_generic_to_shared(sV));
#pragma unroll 4
  for (int it = 0; it < BLK / 8; ++it) {
    const int idx = it * 128 + tid, row = idx >> 4, gran = idx & 15;
    const uint32_t dst = sV_u + (row * kVPitch + gran * 8) * 2;
    if (row < nvis)
      cp_async16(dst, vb + row * row_stride + gran * 8);
    else  // rows past the query get p = 0; keep them finite (0 * NaN would poison O)
      asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(dst), "r"(0) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // K granules for this warp's NT 8-key n-tiles (key row 8*nt + g4)
  uint4 kg[NT][4];
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const int key = warp * KW + q4 * 8 + g4;
    const uint16_t *kr = kb + size_t(min(key, nvis - 1)) * row_stride;
#pragma unroll
    for (int m = 0; m < 4; ++m) kg[q4][m] = ldg_nc_v4(kr + 8 * (c + 4 * m));
  }
  // q A fragments (rows g4 and g4+8; zero beyond R), same d permutation
  uint32_t qa[4][2][2], qb[4][2][2];
  {
    const uint16_t *q0 = a.q + (size_t(b) * a.H + size_t(g) * R + g4) * kHeadDim;
    const uint16_t *q1 = q0 + 8 * kHeadDim;
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint2 v0 = make_uint2(0u, 0u), v1 = make_uint2(0u, 0u);
        if (g4 < R) v0 = *reinterpret_cast<const uint2 *>(q0 + 8 * (c + 4 * m) + 4 * h);
        if (g4 + 8 < R) v1 = *reinterpret_cast<const uint2 *>(q1 + 8 * (c + 4 * m) + 4 * h);
        qa[m][h][0] = v0.x; qa[m][h][1] = v0.y;
        qb[m][h][0] = v1.x; qb[m][h][1] = v1.y;
      }
  }
  // S tiles: acc[q4] = rows (g4, g4+8) x keys (8*nt + 2c, +1)
  float sacc[NT][4];
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[q4][e] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      mma_bf16_16816(sacc[q4], qa[m][0][0], qb[m][0][0], qa[m][0][1], qb[m][0][1], kg[q4][m].x,
                     kg[q4][m].y);
      mma_bf16_16816(sacc[q4], qa[m][1][0], qb[m][1][0], qa[m][1][1], qb[m][1][1], kg[q4][m].z,
                     kg[q4][m].w);
    }
  }
  // mask keys past the query, row max over the block
  float mx0 = -FLT_MAX, mx1 = -FLT_MAX;
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const int k0 = warp * KW + q4 * 8 + 2 * c;
    if (k0 >= nvis) { sacc[q4][0] = -FLT_MAX; sacc[q4][2] = -FLT_MAX; }
    if (k0 + 1 >= nvis) { sacc[q4][1] = -FLT_MAX; sacc[q4][3] = -FLT_MAX; }
    mx0 = fmaxf(mx0, fmaxf(sacc[q4][0], sacc[q4][1]));
    mx1 = fmaxf(mx1, fmaxf(sacc[q4][2], sacc[q4][3]));
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  if (c == 0) { s_m[warp * 16 + g4] = mx0; s_m[warp * 16 + g4 + 8] = mx1; }
  __syncthreads();
  const float m0 = fmaxf(fmaxf(s_m[g4], s_m[16 + g4]), fmaxf(s_m[32 + g4], s_m[48 + g4]));
  const float m1 = fmaxf(fmaxf(s_m[8 + g4], s_m[24 + g4]), fmaxf(s_m[40 + g4], s_m[56 + g4]));
  // P = exp(scale (S - m)), packed straight into A fragments
  uint32_t pa[NT / 2][4];
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const float p0 = exp2f((sacc[q4][0] - m0) * a.scale_log2);
    const float p1 = exp2f((sacc[q4][1] - m0) * a.scale_log2);
    const float p2 = exp2f((sacc[q4][2] - m1) * a.scale_log2);
    const float p3 = exp2f((sacc[q4][3] - m1) * a.scale_log2);
    l0 += p0 + p1;
    l1 += p2 + p3;
    const int kt = q4 >> 1, hi = q4 & 1;   // n-tiles (2kt, 2kt+1) -> k-step kt
    pa[kt][hi ? 2 : 0] = pack_bf16x2(p0, p1);   // row g4
    pa[kt][hi ? 3 : 1] = pack_bf16x2(p2, p3);   // row g4 + 8
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (c == 0) { s_l[warp * 16 + g4] = l0; s_l[warp * 16 + g4 + 8] = l1; }
  // O = P V over this warp's 32 keys (two 16-key k-steps) x 16 d-tiles
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  float oacc[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[dt][e] = 0.f;
#pragma unroll
  for (int kt = 0; kt < NT / 2; ++kt) {
    const int key0 = warp * KW + kt * 16;
#pragma unroll
    for (int dt = 0; dt < 16; dt += 2) {
      // matrices: (keys 0-7, dt), (keys 8-15, dt), (keys 0-7, dt+1), (keys 8-15, dt+1)
      const int mi = lane >> 3, r = lane & 7;
      const int key = key0 + (mi & 1) * 8 + r;
      const int d0 = (dt + (mi >> 1)) * 8;
      uint32_t bv[4];
      ldmatrix_x4_trans(bv, sV_u + (key * kVPitch + d0) * 2);
      mma_bf16_16816(oacc[dt], pa[kt][0], pa[kt][1], pa[kt][2], pa[kt][3], bv[0], bv[1]);
      mma_bf16_16816(oacc[dt + 1], pa[kt][0], pa[kt][1], pa[kt][2], pa[kt][3], bv[2], bv[3]);
    }
  }
  // sum the 4 warps' partial O (rows < R only) and normalise; the partial O
  // area overlays the staged V, so every warp must be done reading V
  __syncthreads();
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int d = dt * 8 + 2 * c;
    if (g4 < R) {
      s_o[(warp * R + g4) * kHeadDim + d] = oacc[dt][0];
      s_o[(warp * R + g4) * kHeadDim + d + 1] = oacc[dt][1];
    }
    if (g4 + 8 < R) {
      s_o[(warp * R + g4 + 8) * kHeadDim + d] = oacc[dt][2];
      s_o[(warp * R + g4 + 8) * kHeadDim + d + 1] = oacc[dt][3];
    }
  }
  __syncthreads();
  for (int x = tid; x < R * kHeadDim; x += 128) {
    const int h = x / kHeadDim, d = x % kHeadDim;
    const float l = s_l[h] + s_l[16 + h] + s_l[32 + h] + s_l[48 + h];
    const float o = s_o[h * kHeadDim + d] + s_o[(R + h) * kHeadDim + d] +
                    s_o[(2 * R + h) * kHeadDim + d] + s_o[(3 * R + h) * kHeadDim + d];
    a.part_o[(prow0 + size_t(h) * a.top_k) * kHeadDim + d] = o / l;
  }
  if (tid < R) {
    const int h = tid;
    const float mh = fmaxf(fmaxf(s_m[h], s_m[16 + h]), fmaxf(s_m[32 + h], s_m[48 + h]));
    const float l = s_l[h] + s_l[16 + h] + s_l[32 + h] + s_l[48 + h];
    a.part_lse[prow0 + size_t(h) * a.top_k] = mh * a.scale + __logf(l);
  }
  dec_merge_if_last<R>(a, b, g);
}

// decode_attn_kernel for FP8 K/V caches: the stored key / value of token s
// (KV head g) is scale[s,g] * E4M3(code).  Same work split as the bf16
// kernel, with these differences:
//   S = q K^T runs in f16 (codes convert exactly; q_idx-style d permutation
//     over 16-code granules, see decode_index_fp8_kernel) and each key's
//     score column is then multiplied by its K scale;
//   V codes are converted (exactly) to bf16 on their way into shared memory,
//     and each key's V scale is folded into P before P is packed to bf16, so
//     the P V MMA is the bf16 one; the row sum uses the unscaled P.
template <int R, int BLK>
__global__ void __launch_bounds__(128) decode_attn_fp8_kernel(const DecodeArgs a) {
  constexpr int KW = BLK / 4;   // keys per warp
  constexpr int NT = KW / 8;    // 8-key n-tiles per warp
  constexpr int NV = BLK / 16;  // 16-code V granules per thread
  extern __shared__ __align__(16) uint8_t dsm[];
  uint16_t *sV = reinterpret_cast<uint16_t *>(dsm);
  float *s_o = reinterpret_cast<float *>(dsm);                     // [4 warps][R rows][128], over V
  float *s_m = reinterpret_cast<float *>(dsm + dec_attn_area<R, BLK>());   // [4][16]
  float *s_l = s_m + 4 * 16;                                        // [4][16]
  const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, c = lane & 3;
  griddep_wait();   // the top-k's selection
  const int n = a.seq_lens[b];
  const int j = (n >= 1 && n <= a.Lmax) ? a.sel[(size_t(b) * a.G + g) * a.top_k + slot] : -1;
  const size_t prow0 = (size_t(b) * a.H + size_t(g) * R) * a.top_k + slot;
  if (j < 0) {   // an unused slot: an empty partial
    if (tid < R) a.part_lse[prow0 + size_t(tid) * a.top_k] = -INFINITY;
    dec_merge_if_last<R>(a, b, g);
    return;
  }
  const int t = n - 1;
  const int nvis = min(BLK, t - j * BLK + 1);
  const size_t tok0 = size_t(b) * a.Lmax + size_t(j) * BLK;   // first token of the block
  const size_t row_stride = size_t(a.G) * kHeadDim;                // codes between tokens
  const uint8_t *kb = a.k8 + (tok0 * a.G + g) * kHeadDim;
  const uint8_t *vb = a.v8 + (tok0 * a.G + g) * kHeadDim;
  const float *ksb = a.k_scale + tok0 * a.G + g;                   // stride G per token
  const float *vsb = a.v_scale + tok0 * a.G + g;
  // V codes: BLK * 8 granules of 16, NV per thread, loaded now and
  // converted into shared memory after S
  uint4 vg[NV];
#pragma unroll
  for (int it = 0; it < NV; ++it) {
    const int idx = it * 128 + tid, row = idx >> 3, gran = idx & 7;
    vg[it] = (row < nvis) ? ldg_nc_v4(vb + row * row_stride + gran * 16) : make_uint4(0, 0, 0, 0);
  }
  // K granules for this warp's NT 8-key n-tiles (key row 8*nt + g4)
  uint4 kg[NT][2];
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const int key = warp * KW + q4 * 8 + g4;
    const uint8_t *kr = kb + size_t(min(key, nvis - 1)) * row_stride;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) kg[q4][gi] = ldg_nc_v4(kr + 16 * (c + 4 * gi));
  }
  // scales of the keys whose S columns this lane holds: 8*nt + 2c, +1
  float ksc[NT][2], vsc[NT][2];
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int key = min(warp * KW + q4 * 8 + 2 * c + e, nvis - 1);
      ksc[q4][e] = __ldg(ksb + size_t(key) * a.G);
      vsc[q4][e] = __ldg(vsb + size_t(key) * a.G);
    }
  // q A fragments in f16 (rows g4 and g4+8; zero beyond R), permuted d
  uint32_t qa[8][2], qb[8][2];
  {
    const uint16_t *q0 = a.q + (size_t(b) * a.H + size_t(g) * R + g4) * kHeadDim;
    const uint16_t *q1 = q0 + 8 * kHeadDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d0 = 16 * (c + 4 * (kk >> 2)) + 4 * (kk & 3);
      uint2 v0 = make_uint2(0u, 0u), v1 = make_uint2(0u, 0u);
      if (g4 < R) v0 = *reinterpret_cast<const uint2 *>(q0 + d0);
      if (g4 + 8 < R) v1 = *reinterpret_cast<const uint2 *>(q1 + d0);
      qa[kk][0] = f16x2_of(bf16_lo(v0.x), bf16_hi(v0.x));
      qa[kk][1] = f16x2_of(bf16_lo(v0.y), bf16_hi(v0.y));
      qb[kk][0] = f16x2_of(bf16_lo(v1.x), bf16_hi(v1.x));
      qb[kk][1] = f16x2_of(bf16_lo(v1.y), bf16_hi(v1.y));
    }
  }
  float sacc[NT][4];
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[q4][e] = 0.f;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const uint32_t wk[4] = {kg[q4][gi].x, kg[q4][gi].y, kg[q4][gi].z, kg[q4][gi].w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int kk = 4 * gi + w;
        mma_f16_16816(sacc[q4], qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1],
                      e4m3x2_to_f16x2(wk[w]), e4m3x2_to_f16x2(wk[w] >> 16));
      }
    }
    sacc[q4][0] *= ksc[q4][0]; sacc[q4][2] *= ksc[q4][0];
    sacc[q4][1] *= ksc[q4][1]; sacc[q4][3] *= ksc[q4][1];
  }
  // V codes -> bf16 rows in shared memory (rows past the query are zero)
#pragma unroll
  for (int it = 0; it < NV; ++it) {
    const int idx = it * 128 + tid, row = idx >> 3, gran = idx & 7;
    const uint32_t wv[4] = {vg[it].x, vg[it].y, vg[it].z, vg[it].w};
    uint32_t o[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t h = e4m3x2_to_f16x2(wv[w] >> (16 * hh));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
        o[2 * w + hh] = pack_bf16x2(f.x, f.y);
      }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(sV + row * kVPitch + gran * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // mask keys past the query, row max over the block
  float mx0 = -FLT_MAX, mx1 = -FLT_MAX;
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const int k0 = warp * KW + q4 * 8 + 2 * c;
    if (k0 >= nvis) { sacc[q4][0] = -FLT_MAX; sacc[q4][2] = -FLT_MAX; }
    if (k0 + 1 >= nvis) { sacc[q4][1] = -FLT_MAX; sacc[q4][3] = -FLT_MAX; }
    mx0 = fmaxf(mx0, fmaxf(sacc[q4][0], sacc[q4][1]));
    mx1 = fmaxf(mx1, fmaxf(sacc[q4][2], sacc[q4][3]));
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  if (c == 0) { s_m[warp * 16 + g4] = mx0; s_m[warp * 16 + g4 + 8] = mx1; }
  __syncthreads();   // also: the staged V rows are complete
  const float m0 = fmaxf(fmaxf(s_m[g4], s_m[16 + g4]), fmaxf(s_m[32 + g4], s_m[48 + g4]));
  const float m1 = fmaxf(fmaxf(s_m[8 + g4], s_m[24 + g4]), fmaxf(s_m[40 + g4], s_m[56 + g4]));
  // P = exp(scale (S - m)); the A fragments carry P * (V scale of the key)
  uint32_t pa[NT / 2][4];
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int q4 = 0; q4 < NT; ++q4) {
    const float p0 = exp2f((sacc[q4][0] - m0) * a.scale_log2);
    const float p1 = exp2f((sacc[q4][1] - m0) * a.scale_log2);
    const float p2 = exp2f((sacc[q4][2] - m1) * a.scale_log2);
    const float p3 = exp2f((sacc[q4][3] - m1) * a.scale_log2);
    l0 += p0 + p1;
    l1 += p2 + p3;
    const int kt = q4 >> 1, hi = q4 & 1;
    pa[kt][hi ? 2 : 0] = pack_bf16x2(p0 * vsc[q4][0], p1 * vsc[q4][1]);   // row g4
    pa[kt][hi ? 3 : 1] = pack_bf16x2(p2 * vsc[q4][0], p3 * vsc[q4][1]);   // row g4 + 8
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (c == 0) { s_l[warp * 16 + g4] = l0; s_l[warp * 16 + g4 + 8] = l1; }
  const uint32_t sV_u = static_cast<uint32_t>(__cvta_generic_to_shared(sV));
  float oacc[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[dt][e] = 0.f;
#pragma unroll
  for (int kt = 0; kt < NT / 2; ++kt) {
    const int key0 = warp * KW + kt * 16;
#pragma unroll
    for (int dt = 0; dt < 16; dt += 2) {
      const int mi = lane >> 3, r = lane & 7;
      const int key = key0 + (mi & 1) * 8 + r;
      const int d0 = (dt + (mi >> 1)) * 8;
      uint32_t bv[4];
      ldmatrix_x4_trans(bv, sV_u + (key * kVPitch + d0) * 2);
      mma_bf16_16816(oacc[dt], pa[kt][0], pa[kt][1], pa[kt][2], pa[kt][3], bv[0], bv[1]);
      mma_bf16_16816(oacc[dt + 1], pa[kt][0], pa[kt][1], pa[kt][2], pa[kt][3], bv[2], bv[3]);
    }
  }
  __syncthreads();   // the partial O area overlays the staged V: all warps done with V
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int d = dt * 8 + 2 * c;
    if (g4 < R) {
      s_o[(warp * R + g4) * kHeadDim + d] = oacc[dt][0];
      s_o[(warp * R + g4) * kHeadDim + d + 1] = oacc[dt][1];
    }
    if (g4 + 8 < R) {
      s_o[(warp * R + g4 + 8) * kHeadDim + d] = oacc[dt][2];
      s_o[(warp * R + g4 + 8) * kHeadDim + d + 1] = oacc[dt][3];
    }
  }
  __syncthreads();
  for (int x = tid; x < R * kHeadDim; x += 128) {
    const int h = x / kHeadDim, d = x % kHeadDim;
    const float l = s_l[h] + s_l[16 + h] + s_l[32 + h] + s_l[48 + h];
    const float o = s_o[h * kHeadDim + d] + s_o[(R + h) * kHeadDim + d] +
                    s_o[(2 * R + h) * kHeadDim + d] + s_o[(3 * R + h) * kHeadDim + d];
    a.part_o[(prow0 + size_t(h) * a.top_k) * kHeadDim + d] = o / l;
  }
  if (tid < R) {
    const int h = tid;
    const float mh = fmaxf(fmaxf(s_m[h], s_m[16 + h]), fmaxf(s_m[32 + h], s_m[48 + h]));
    const float l = s_l[h] + s_l[16 + h] + s_l[32 + h] + s_l[48 + h];
    a.part_lse[prow0 + size_t(h) * a.top_k] = mh * a.scale + __logf(l);
  }
  dec_merge_if_last<R>(a, b, g);
}

// Launch as a programmatic dependent of the previous kernel in the stream.
template <typename Kern>
cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             const DecodeArgs &a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int R, int BLK>
cudaError_t launch_decode_attn(const DecodeArgs &a, cudaStream_t st) {
  constexpr int smem = dec_attn_smem<R, BLK>();
  auto kern = a.k8 ? decode_attn_fp8_kernel<R, BLK> : decode_attn_kernel<R, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(kern, dim3(a.top_k, a.G, a.B), dim3(128), smem, st, a);
}

template <int BLK>
cudaError_t launch_decode_b(const DecodeArgs &a, cudaStream_t st) {
  // the scan: one warp per 128-key chunk, 8 chunks per CTA
  const int chunks = (a.Lmax + 127) / 128;
  const dim3 gi((chunks + 7) / 8, a.B);
  if (a.k_idx8) {
    if (a.d_idx == 64)
      decode_index_fp8_kernel<64, BLK><<<gi, 256, 0, st>>>(a);
    else
      decode_index_fp8_kernel<128, BLK><<<gi, 256, 0, st>>>(a);
  } else if (a.d_idx == 64) {
    decode_index_kernel<64, BLK><<<gi, 256, 0, st>>>(a);
  } else {
    decode_index_kernel<128, BLK><<<gi, 256, 0, st>>>(a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_dependent(decode_topk_kernel, dim3(a.B * a.G), dim3(kTopkWarps * 32), 0, st, a);
  if (e != cudaSuccess) return e;
  switch (a.H / a.G) {
    case 1: e = launch_decode_attn<1, BLK>(a, st); break;
    case 2: e = launch_decode_attn<2, BLK>(a, st); break;
    case 4: e = launch_decode_attn<4, BLK>(a, st); break;
    case 8: e = launch_decode_attn<8, BLK>(a, st); break;
    case 16: e = launch_decode_attn<16, BLK>(a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  return a.blk == 64 ? launch_decode_b<64>(a, st) : launch_decode_b<128>(a, st);
}

}  // namespace msa
