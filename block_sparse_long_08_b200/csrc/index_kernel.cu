// Index Branch on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every query t and GQA group g, the block scores
//   S[b,g,t,j] = max_{s in block j} q_idx[b,t,g] . k_idx[b,s]      (j < t/128)
// ("MiniMax M3 sparse attention" explainer, mlqm.cn/news/533796, §2.1: one
// index query per group, one shared index key, Block Max Pooling), and either
// stores them (SCORES mode) or keeps, per row, a running top-(top_k-1) list
// and writes the selection with the forced local block (FUSED mode;
// researchpapers.dev "MiniMax Sparse Attention", section "机制").
//
// Causality needs no element mask: the local block b_t is always selected,
// so only blocks j < b_t are scored, and every such block is entirely
// visible.  For a 128-query tile i the work is the tile row of 128-key
// chunks j = 0..i-1.  With 64-token blocks (BLK = 64) a chunk holds two
// blocks, pooled separately, and the tile's second half (rows 64..127, local
// block 2i+1) also scores block 2i, the first half of chunk i.
//
// Kernel structure (persistent, one CTA per SM, 12 warps = 3 warpgroups):
//   warp 0    TMA producer: the tile's q_idx rows for GP groups (resident),
//             then k_idx blocks two at a time into an NS-deep ring.
//   warp 1    TMEM owner + MMA issuer: per (stage, group) one
//             M=128 x N=256 x K=d_idx UMMA into one of two TMEM accumulators.
//   warps 2-3 idle (they complete the first warpgroup).
//   warps 4-11 epilogue, two sets of four warps (one warp per TMEM lane
//             quadrant).  Set h reads key block h (columns 128h..128h+127)
//             of every accumulator: thread r owns row r (one query), loads
//             its 128 columns in one TMEM round trip, frees the accumulator,
//             max-pools the block and stores the score or inserts it into
//             a register-resident sorted list.  At the end of a tile the two
//             sets' lists (even / odd blocks) are merged through shared
//             memory.
// The TMEM accumulator is freed as soon as its columns sit in registers, so
// the next UMMA into that slot waits one TMEM round trip, not the max-pool
// and list work.  The first warpgroup gives registers to the epilogue
// warpgroups (setmaxnreg: 3 x 128 x 168 = 128 x 56 + 256 x 224).
// One k_idx stage feeds GP groups, which halves L2->SM traffic for GP = 2.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace msa {

namespace {

template <int DI, int GP, int KCAP>
struct IndexCfg {
  static constexpr int NCH = DI / 64;                 // 128-B K chunks per row
  static constexpr int Q_BYTES = GP * NCH * 16384;    // resident q_idx tiles
  static constexpr int STAGE_BYTES = NCH * 2 * 16384; // two k_idx blocks
  static constexpr int MERGE_BYTES = GP * KCAP * 128 * 8;  // list exchange
  static constexpr int NS_RAW = (232448 - 1280 - MERGE_BYTES - Q_BYTES) / STAGE_BYTES;
  static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;
  static constexpr int BAR_OFF = Q_BYTES + NS * STAGE_BYTES;
  static constexpr int MERGE_OFF = BAR_OFF + 256;
  static constexpr int SMEM = MERGE_OFF + MERGE_BYTES + 1024;  // + align slack
  static constexpr int THREADS = 384;
  static_assert(NS >= 2, "k_idx ring needs two stages");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Register split between the warpgroups: the launch gives every thread 168
// registers (384 threads); the producer/MMA warpgroup keeps 56 and the two
// epilogue warpgroups take 224 (128*56 + 256*224 = 384*168).
__device__ __forceinline__ void regs_dec_56() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
}
__device__ __forceinline__ void regs_inc_224() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
}
__device__ __forceinline__ void epi_bar_sync() {  // the 8 epilogue warps
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

struct IndexWork {
  int i, b, gp, stages;
};

template <int BLK>
__device__ __forceinline__ IndexWork index_work(const IndexArgs &a, int u, int GPn) {
  const int ngp = a.G / GPn;
  IndexWork w;
  if (a.items) {   // ragged batch: the host's (b, i) list, every group pair of each
    const int2 it = a.items[u / ngp];
    w.b = it.x;
    w.i = it.y;
    w.gp = u % ngp;
  } else {
    w.i = a.i_hi - 1 - u / (a.B * ngp);
    const int rem = u % (a.B * ngp);
    w.b = rem / ngp;
    w.gp = rem % ngp;
  }
  // largest local block among the tile's rows; chunks 0..i-1 (BLK 128) or
  // 0..i (BLK 64) hold every block a row of the tile may score
  const int max_bt = (BLK == 128) ? w.i : 2 * w.i + 1;
  const bool need = a.write_scores ? (max_bt >= 1) : (max_bt >= a.top_k && a.top_k >= 2);
  w.stages = need ? ((BLK == 128) ? (w.i + 1) / 2 : w.i / 2 + 1) : 0;
  return w;
}

// Selection / score row of position t of the item's sequence for group g,
// or -1 when t is not one of the launch's query rows.
__device__ __forceinline__ long long index_out_row(const IndexArgs &a, const int4 &s, int g,
                                                   int t) {
  const int tl = t - s.y;
  const int r = s.x + tl;
  if (tl < 0 || tl >= s.z || r < a.r_lo || r >= a.r_hi) return -1;
  return (long long)s.w + (long long)g * a.q.sel_gs + tl;
}

// Work item of this CTA in round r (snake order over CTAs; items are sorted
// by decreasing tile row length, so consecutive rounds balance out).
__device__ __forceinline__ int index_item(int r, int n_items) {
  const int u = r * gridDim.x + ((r & 1) ? (gridDim.x - 1 - blockIdx.x) : blockIdx.x);
  return u < n_items ? u : -1;
}

template <int KCAP>
__device__ __forceinline__ void list_insert(float (&ls)[KCAP], int (&lj)[KCAP], float s, int j) {
  // Insert (s, j) into the list kept in (score desc, id asc) order, for ids
  // in any order (the merge of the two sets' lists).  The carried entry is
  // compared lexicographically, so an entry pushed down by the insertion
  // keeps its place ahead of an equal-score entry with a higher id.
  float cs = s;
  int cj = j;
#pragma unroll
  for (int k = 0; k < KCAP; ++k) {
    const bool sw = (cs > ls[k]) || (cs == ls[k] && cj < lj[k]);
    const float ts = ls[k];
    const int tj = lj[k];
    ls[k] = sw ? cs : ts;
    lj[k] = sw ? cj : tj;
    cs = sw ? ts : cs;
    cj = sw ? tj : cj;
  }
}

template <int KCAP>
__device__ __forceinline__ void list_insert_tail(float (&ls)[KCAP], int (&lj)[KCAP], float s, int j) {
  // Insert (s, j) when j is above every kept id (the blocks of one epilogue
  // set arrive in increasing id order): a kept entry ranks ahead of the new
  // one exactly when its score is >= s, so the insertion point is the number
  // of such entries and every slot is updated independently -- no carried
  // compare chain.  Walking k downwards reads ls[k-1] before it is replaced.
  bool ge[KCAP];
#pragma unroll
  for (int k = 0; k < KCAP; ++k) ge[k] = ls[k] >= s;
#pragma unroll
  for (int k = KCAP - 1; k >= 1; --k) {
    ls[k] = ge[k] ? ls[k] : (ge[k - 1] ? s : ls[k - 1]);
    lj[k] = ge[k] ? lj[k] : (ge[k - 1] ? j : lj[k - 1]);
  }
  ls[0] = ge[0] ? ls[0] : s;
  lj[0] = ge[0] ? lj[0] : j;
}

template <int KCAP>
__device__ __forceinline__ void sort_ids_asc(int (&v)[KCAP]) {
  // Bitonic network over KCAP (power of two) register values.
#pragma unroll
  for (int k = 2; k <= KCAP; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int x = 0; x < KCAP; ++x) {
        const int y = x ^ j;
        if (y > x) {
          const bool up = (x & k) == 0;
          const int lo = min(v[x], v[y]), hi = max(v[x], v[y]);
          v[x] = up ? lo : hi;
          v[y] = up ? hi : lo;
        }
      }
    }
  }
}

// Max over 2 x 32 fp32 values (two independent chains).
__device__ __forceinline__ float max2x32(const float (&a)[32], const float (&b)[32]) {
  float m0 = max3f(a[0], a[1], a[2]), m1 = max3f(b[0], b[1], b[2]);
#pragma unroll
  for (int x = 3; x + 2 <= 31; x += 2) {
    m0 = max3f(m0, a[x], a[x + 1]);
    m1 = max3f(m1, b[x], b[x + 1]);
  }
  return fmaxf(fmaxf(m0, a[31]), fmaxf(m1, b[31]));
}

// Max over 4 x 32 fp32 values with three-input max (4 independent chains).
__device__ __forceinline__ float max4x32(const float (&a)[32], const float (&b)[32],
                                         const float (&c)[32], const float (&d)[32]) {
  float m0 = max3f(a[0], a[1], a[2]), m1 = max3f(b[0], b[1], b[2]);
  float m2 = max3f(c[0], c[1], c[2]), m3 = max3f(d[0], d[1], d[2]);
#pragma unroll
  for (int x = 3; x + 2 <= 31; x += 2) {
    m0 = max3f(m0, a[x], a[x + 1]);
    m1 = max3f(m1, b[x], b[x + 1]);
    m2 = max3f(m2, c[x], c[x + 1]);
    m3 = max3f(m3, d[x], d[x + 1]);
  }
  m0 = fmaxf(m0, a[31]);
  m1 = fmaxf(m1, b[31]);
  m2 = fmaxf(m2, c[31]);
  m3 = fmaxf(m3, d[31]);
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// One block score of a row: stored (SCORES mode) or offered to the row's
// running list (FUSED mode; ids arrive in increasing order within a set).
template <int KCAP>
__device__ __forceinline__ void put_score(const IndexArgs &a, const int4 &sq, int g, int t,
                                          float (&ls)[KCAP], int (&lj)[KCAP], float sc, int jb) {
  if (a.write_scores) {
    const long long orow = index_out_row(a, sq, g, t);
    if (orow >= 0) a.scores[orow * a.nb + jb] = sc;
  } else if (sc > ls[KCAP - 1]) {
    list_insert_tail<KCAP>(ls, lj, sc, jb);
  }
}

template <int DI, int GP, int KCAP, int BLK>
__global__ void __launch_bounds__(384, 1)
    msa_index_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, const IndexArgs a) {
  using C = IndexCfg<DI, GP, KCAP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t s_q = smem_u32(smem);
  const uint32_t s_k = s_q + C::Q_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  // barrier slots
  const uint32_t b_qfull = smem_u32(&bars[0]);
  const uint32_t b_qempty = smem_u32(&bars[1]);
  const uint32_t b_kfull = smem_u32(&bars[2]);            // + 8*s
  const uint32_t b_kempty = smem_u32(&bars[2 + C::NS]);   // + 8*s
  const uint32_t b_accfull = smem_u32(&bars[2 + 2 * C::NS]);   // + 8*slot
  const uint32_t b_accempty = smem_u32(&bars[4 + 2 * C::NS]);  // + 8*slot
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(&bars[8 + 2 * C::NS]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_kfull + 8 * s, 1);
      mbar_init(b_kempty + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_accfull + 8 * s, 1);
      mbar_init(b_accempty + 8 * s, 8);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp < 4) {
   // setmaxnreg is warpgroup-wide: all four warps of warpgroup 0 execute
   // this one instruction, then split into their roles.
   regs_dec_56();
   if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      int kst = 0;
      uint32_t kph = 0, qph = 0;
      for (int r = 0;; ++r) {
        const int u = index_item(r, a.n_items);
        if (u < 0) break;
        const IndexWork w = index_work<BLK>(a, u, GP);
        if (w.stages == 0) continue;
        if (!mbar_wait(b_qempty, qph ^ 1, abort_flag, a.status)) break;
        qph ^= 1;
        mbar_arrive_expect_tx(b_qfull, C::Q_BYTES);
        // the tile's q_idx rows (rows outside the sequence load as zeros or
        // another sequence's values; their results are never written)
        const int4 sq = qgeo_seq(a.q, w.b);
        for (int gi = 0; gi < GP; ++gi)
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(s_q + (gi * C::NCH + c) * 16384, &tm_q, b_qfull, c * 64, w.gp * GP + gi,
                        sq.x + w.i * 128 - sq.y);
        bool ok = true;
        for (int s = 0; s < w.stages; ++s) {
          if (!mbar_wait(b_kempty + 8 * kst, kph ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(b_kfull + 8 * kst, C::STAGE_BYTES);
          const uint32_t dst = s_k + kst * C::STAGE_BYTES;
          const int row0 = w.b * a.L + (2 * s) * 128;   // 128-key chunks 2s, 2s+1
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_2d(dst + c * 32768, &tm_k, b_kfull + 8 * kst, c * 64, row0);
            tma_load_2d(dst + c * 32768 + 16384, &tm_k, b_kfull + 8 * kst, c * 64, row0 + 128);
          }
          if (++kst == C::NS) { kst = 0; kph ^= 1; }
        }
        if (!ok) break;
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, 0, 0);
      int kst = 0;
      uint32_t kph = 0, qph = 0;
      uint32_t jc = 0;
      for (int r = 0;; ++r) {
        const int u = index_item(r, a.n_items);
        if (u < 0) break;
        const IndexWork w = index_work<BLK>(a, u, GP);
        if (w.stages == 0) continue;
        if (!mbar_wait(b_qfull, qph, abort_flag, a.status)) break;
        qph ^= 1;
        tc_fence_after();
        bool ok = true;
        for (int s = 0; s < w.stages && ok; ++s) {
          if (!mbar_wait(b_kfull + 8 * kst, kph, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = s_k + kst * C::STAGE_BYTES;
          for (int gi = 0; gi < GP; ++gi) {
            const uint32_t slot = jc & 1;
            if (!mbar_wait(b_accempty + 8 * slot, ((jc >> 1) & 1) ^ 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + slot * 256;
#pragma unroll
            for (int kk = 0; kk < DI / 16; ++kk) {
              const int c = kk >> 2;
              const uint32_t off = (kk & 3) * 32;
              const uint64_t ad = sdesc_sw128(s_q + (gi * C::NCH + c) * 16384 + off, 16, 1024);
              const uint64_t bd = sdesc_sw128(kbase + c * 32768 + off, 16, 1024);
              umma_f16_ss(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            umma_commit(b_accfull + 8 * slot);
            ++jc;
          }
          umma_commit(b_kempty + 8 * kst);
          if (++kst == C::NS) { kst = 0; kph ^= 1; }
        }
        umma_commit(b_qempty);
        if (!ok) break;
      }
    }
   }  // warps 2-3: idle
  } else {
    // ------------------------------------------------------------ epilogue
    regs_inc_224();  // the same instruction for both epilogue warpgroups
    const int eset = (warp - 4) >> 2;          // key block h = eset of each job
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (uint32_t(quad * 32) << 16);
    const int k1 = a.top_k - 1;
    // Slots [0, KCAP-k1) hold sentinels (+inf, id -1) that rank ahead of
    // every block and never move; the kept entries occupy the last k1 slots,
    // so the worst kept score is always ls[KCAP-1].
    const int n_sent = KCAP - k1;
    float *m_score = reinterpret_cast<float *>(smem + C::MERGE_OFF);
    int *m_id = reinterpret_cast<int *>(smem + C::MERGE_OFF + C::MERGE_BYTES / 2);
    uint32_t jc = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = index_item(r, a.n_items);
      if (u < 0) break;
      const IndexWork w = index_work<BLK>(a, u, GP);
      const int t = w.i * 128 + row;   // query tiles hold 128 queries whatever the block
      const int bt = t / BLK;          // this row's local block
      const int4 sq = qgeo_seq(a.q, w.b);
      float ls[GP][KCAP];
      int lj[GP][KCAP];
#pragma unroll
      for (int gi = 0; gi < GP; ++gi) {
#pragma unroll
        for (int k = 0; k < KCAP; ++k) {
          ls[gi][k] = k < n_sent ? INFINITY : -FLT_MAX;
          lj[gi][k] = k < n_sent ? -1 : INT_MAX;
        }
      }
      for (int s = 0; s < w.stages && ok; ++s) {
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) {
          const uint32_t slot = jc & 1;
          if (!mbar_wait(b_accfull + 8 * slot, (jc >> 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int j = 2 * s + eset;   // 128-key chunk
          // warp-uniform: a warp's rows are all below or all above 64
          const bool use = (BLK == 128) ? (j < w.i) : (j < w.i || (j == w.i && row >= 64));
          float v0[32], v1[32], v2[32], v3[32];
          if (use) {
            const uint32_t ta = lane_base + slot * 256 + eset * 128;
            tmem_ld32(ta, v0);
            tmem_ld32(ta + 32, v1);
            tmem_ld32(ta + 64, v2);
            tmem_ld32(ta + 96, v3);
            tmem_wait_ld();
          }
          // the accumulator is in registers: hand the slot back to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_accempty + 8 * slot);
          ++jc;
          if (use) {
            if (BLK == 128) {
              put_score<KCAP>(a, sq, w.gp * GP + gi, t, ls[gi], lj[gi], max4x32(v0, v1, v2, v3), j);
            } else {
              // blocks 2j (columns 0..63) and 2j+1 (64..127); block 2i+1 is
              // a local block, never scored
              put_score<KCAP>(a, sq, w.gp * GP + gi, t, ls[gi], lj[gi], max2x32(v0, v1), 2 * j);
              if (j < w.i)
                put_score<KCAP>(a, sq, w.gp * GP + gi, t, ls[gi], lj[gi], max2x32(v2, v3),
                                2 * j + 1);
            }
          }
        }
      }
      // After a failed wait, items without a merge end here; an item with a
      // merge still meets the other set at both barriers below, then every
      // epilogue warp leaves together.
      if (a.write_scores) {
        if (!ok) break;
        if (eset == 0) {
#pragma unroll
          for (int gi = 0; gi < GP; ++gi) {
            const long long orow = index_out_row(a, sq, w.gp * GP + gi, t);
            if (orow < 0) continue;
            float *dst = a.scores + orow * a.nb;
            for (int j = bt; j < a.nb; ++j) dst[j] = -INFINITY;
          }
        }
        continue;
      }
      if (((BLK == 128) ? w.i : 2 * w.i + 1) + 1 <= a.top_k) {   // every row keeps all its blocks
        if (!ok) break;
        if (eset == 0) {
#pragma unroll
          for (int gi = 0; gi < GP; ++gi) {
            const long long orow = index_out_row(a, sq, w.gp * GP + gi, t);
            if (orow < 0) continue;
            int32_t *dst = a.sel + orow * a.top_k;
            for (int k = 0; k < a.top_k; ++k) dst[k] = (k <= bt) ? k : -1;
          }
        }
        continue;
      }
      // merge the odd-block lists (set 1) into the even-block lists (set 0)
      if (eset == 1) {
#pragma unroll
        for (int gi = 0; gi < GP; ++gi)
#pragma unroll
          for (int k = 0; k < KCAP; ++k) {
            m_score[(gi * KCAP + k) * 128 + row] = ls[gi][k];
            m_id[(gi * KCAP + k) * 128 + row] = lj[gi][k];
          }
      }
      epi_bar_sync();
      const bool abort_now = (*abort_flag != 0);   // the same value for all 8 warps
      if (eset == 0 && !abort_now) {
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) {
#pragma unroll
          for (int k = 0; k < KCAP; ++k) {
            const float sc = m_score[(gi * KCAP + k) * 128 + row];
            const int id = m_id[(gi * KCAP + k) * 128 + row];
            if (id >= 0 && id != INT_MAX) list_insert<KCAP>(ls[gi], lj[gi], sc, id);
          }
          const long long orow = index_out_row(a, sq, w.gp * GP + gi, t);
          if (orow < 0) continue;
          int32_t *dst = a.sel + orow * a.top_k;
          if (bt + 1 <= a.top_k) {   // (BLK 64) this half of the tile keeps all its blocks
            for (int k = 0; k < a.top_k; ++k) dst[k] = (k <= bt) ? k : -1;
            continue;
          }
          int ids[KCAP];
#pragma unroll
          for (int k = 0; k < KCAP; ++k) ids[k] = (k >= n_sent) ? lj[gi][k] : INT_MAX;
          sort_ids_asc<KCAP>(ids);
          if ((a.top_k & 3) == 0) {
#pragma unroll
            for (int k = 0; k < KCAP; k += 4) {
              if (k < a.top_k) {
                int4 o;
                o.x = (k + 0 < k1) ? ids[k + 0] : (k + 0 == k1 ? bt : -1);
                o.y = (k + 1 < k1) ? ids[k + 1] : (k + 1 == k1 ? bt : -1);
                o.z = (k + 2 < k1) ? ids[k + 2] : (k + 2 == k1 ? bt : -1);
                o.w = (k + 3 < k1) ? ids[k + 3] : (k + 3 == k1 ? bt : -1);
                *reinterpret_cast<int4 *>(dst + k) = o;
              }
            }
          } else {
            // top_k can be KCAP + 1 (k1 == KCAP): the local block takes slot KCAP
#pragma unroll
            for (int k = 0; k <= KCAP; ++k)
              if (k < a.top_k)
                dst[k] = (k < k1) ? ids[k < KCAP ? k : KCAP - 1] : (k == k1 ? bt : -1);
          }
        }
      }
      epi_bar_sync();   // set 1 may overwrite the exchange area next tile
      if (abort_now) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int DI, int GP, int KCAP, int BLK>
cudaError_t launch_index_t(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                           int num_sms, cudaStream_t st) {
  using C = IndexCfg<DI, GP, KCAP>;
  auto kern = msa_index_kernel<DI, GP, KCAP, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  kern<<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, a);
  return cudaGetLastError();
}

template <int DI, int GP, int BLK>
cudaError_t launch_index_k(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                           int num_sms, cudaStream_t st) {
  const int k1 = a.top_k - 1;
  if (k1 <= 4) return launch_index_t<DI, GP, 4, BLK>(tq, tk, a, num_sms, st);
  if (k1 <= 8) return launch_index_t<DI, GP, 8, BLK>(tq, tk, a, num_sms, st);
  return launch_index_t<DI, GP, 16, BLK>(tq, tk, a, num_sms, st);
}

template <int BLK>
cudaError_t launch_index_b(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                           int num_sms, cudaStream_t st) {
  const int gp = index_groups_per_cta(a.G, a.top_k);
  if (a.top_k - 1 > 16) {
    // wide lists: one group per CTA, 32-entry list
    if (a.d_idx == 64) return launch_index_t<64, 1, 32, BLK>(tq, tk, a, num_sms, st);
    return launch_index_t<128, 1, 32, BLK>(tq, tk, a, num_sms, st);
  }
  if (a.d_idx == 64)
    return gp == 2 ? launch_index_k<64, 2, BLK>(tq, tk, a, num_sms, st)
                   : launch_index_k<64, 1, BLK>(tq, tk, a, num_sms, st);
  return gp == 2 ? launch_index_k<128, 2, BLK>(tq, tk, a, num_sms, st)
                 : launch_index_k<128, 1, BLK>(tq, tk, a, num_sms, st);
}

}  // namespace

int index_groups_per_cta(int G, int top_k) { return (G % 2 == 0 && top_k - 1 <= 16) ? 2 : 1; }

cudaError_t launch_index_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                                int num_sms, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  if (a.blk == 64) return launch_index_b<64>(tq, tk, a, num_sms, st);
  return launch_index_b<128>(tq, tk, a, num_sms, st);
}

}  // namespace msa
