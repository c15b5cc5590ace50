// Main Branch, prefill: exact softmax attention over the selected blocks,
// organised key-block-outer ("MiniMax M3 sparse attention" explainer,
// mlqm.cn/news/533796, §2.2: gather the selected K/V blocks and run ordinary
// attention, all heads of a group sharing one selection; researchpapers.dev
// "MiniMax Sparse Attention", sections "机制" and "对工程团队的意义": query
// gathering and a reverse index; baguaai.com 稀疏注意力 MSA entry: "KV
// external aggregation Q").
//
// One work item = one (b, g, key block j) and up to 128/R queries that
// selected j, each with its R heads: a 128-row tile.  Blocks hold BLK = 128
// or 64 keys (the explainer's §4.2 reasons with 64-token blocks).  Per item:
//   S = Q K_j^T   (UMMA M=128, N=BLK, K=128, fp32 in TMEM)
//   softmax       row r: mask s <= t (only on the diagonal block), row max,
//                 exp2, row sum, P as bf16 pairs back into S's TMEM columns
//   O = P V_j     (UMMA with A = P read from TMEM, V consumed MN-major
//                 straight from its TMA tile)
//   partial       O / l (bf16) and lse = ln(sum exp(scale q.k)) per row; a
//                 second kernel merges a query row's <= top_k partials.
//
// The work is HBM-bound: per item 32 KB of gathered q rows come in and 32 KB
// of partials go out, against 0.5 us of tensor work.  The kernel is built to
// keep those transfers in flight (one persistent CTA per SM, 16 warps with
// fixed roles):
//   warp 0     K/V producer: TMA loads of K_j and V_j into a ring of 32 KB
//              tiles, once per run of consecutive items with the same key
//              block (items are ordered by (b, g, j)).
//   warp 1     TMEM owner and MMA issuer: issues S_i and O_i in whatever
//              order their inputs become ready (non-blocking barrier probes).
//   warps 2-7  the gather team (192 threads) takes every item in turn: it
//              publishes the item's query list and gathers the q rows (R
//              heads of a query are 256*R contiguous bytes) with cp.async
//              into a free stage's 128B-swizzled tile.
//   warps 8-15 two softmax warpgroups, even and odd items, each with its own
//              TMEM slot: 128 columns for S (then P over its first BLK/2
//              columns) and 128 for O; 512 columns in all.  After the softmax
//              a group loads O, stages the bf16 partial rows in the item's
//              stage and writes them with one bulk copy per warp.
// A stage holds Q, then the staged partial of one item; with NQ stages the
// q gather of item i+NQ starts as soon as item i's partial has left.  Seven
// 32 KB tiles are split between stages and K/V tiles (AttnCfg).  P goes
// through TMEM rather than shared memory: it saves the softmax 2048 16-byte
// shared stores per item and the UMMA a 32 KB shared-memory read, and the
// SM's shared-memory instruction path is what sets the item period.
//
// Partial layout.  The partials of a chunk are indexed by reverse-index list
// position: the entry at position pos (query t, slot k of group g) owns rows
// pos*R + hh (hh < R), so an item's rows are one contiguous range and leave
// in one bulk copy.  Inside a row of 16 granules of 16 bytes, granule c is
// stored at granule c ^ (row & 7): the staging writes are then free of bank
// conflicts, and the merge undoes the permutation when it reads.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kAttnThreads = 512;
constexpr int kTile = 32768;                         // 128 rows x 256 B

// Shared-memory plan per head ratio R.  Seven 32 KB tiles: NQ Q/partial
// stages and NKV K/V tiles.  Four stages (with three K/V tiles, enough when
// items of one key block come in runs) for R >= 2; for R = 1 the 128-entry
// item lists leave room for three stages only, with four K/V tiles.
template <int R>
struct AttnCfg {
  static constexpr int QPI = 128 / R;                 // queries per item
  static constexpr int NQ = (R == 1) ? 3 : 4;
  static constexpr int NKV = 7 - NQ;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = NQ * kTile;
  static constexpr int SMEM_CTL = SMEM_KV + NKV * kTile;   // 229376
  // mbarrier slots (8 bytes each) at SMEM_CTL
  static constexpr int BAR_QFULL = 0;                 // [NQ]  gather team copies + list
  static constexpr int BAR_STEMPTY = NQ;              // [NQ]  four storing warps
  static constexpr int BAR_KVFULL = 2 * NQ;           // [NKV] TMA transaction bytes
  static constexpr int BAR_KVEMPTY = 2 * NQ + NKV;    // [NKV] UMMA commit
  static constexpr int BAR_SFULL = 2 * NQ + 2 * NKV;  // [2]   UMMA commit
  static constexpr int BAR_PFULL = BAR_SFULL + 2;     // [2]   128 softmax threads
  static constexpr int BAR_OFULL = BAR_PFULL + 2;     // [2]   UMMA commit
  static constexpr int BAR_TMEMPTY = BAR_OFULL + 2;   // [2]   128 softmax threads
  static constexpr int BAR_DRAIN = BAR_TMEMPTY + 2;   // UMMA commit on the way out
  static constexpr int NUM_BARS = BAR_DRAIN + 1;
  static constexpr int CTL_MISC = NUM_BARS * 8;       // tmem holder, abort flag
  static constexpr int CTL_DESC = (CTL_MISC + 8 + 15) & ~15;   // [NQ] int4 {bgj, start, n, -}
  static constexpr int CTL_PRE = CTL_DESC + 16 * NQ;  // int4: the gather team's next item
  static constexpr int CTL_LIST = CTL_PRE + 16;       // [NQ][QPI] list entries
  static constexpr int CTL_BYTES = CTL_LIST + NQ * QPI * 4;
  static constexpr int SMEM = SMEM_CTL + CTL_BYTES + 1024;   // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32 pair arithmetic (one instruction for two lanes of data).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}


// Register split: the launch gives 128 registers to each of the 512 threads;
// warpgroups 0-1 (producer, MMA, gatherers) keep 64 and the two softmax
// warpgroups take 184 (256*64 + 256*184 = 63488 <= 65536).
__device__ __forceinline__ void regs_dec_64() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
}
__device__ __forceinline__ void regs_inc_184() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
}

// Position of one thread in the item list of its CTA: item w belongs to the
// key block bgj with item_off[bgj] <= w < item_off[bgj+1].
struct ItemWalk {
  int wb, it_lo, it_hi, l_lo, l_hi;
  __device__ void init(const AttnArgs &a, int n_bgj, int w) {
    int lo = 0, hi = n_bgj - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.item_off[mid] <= w) lo = mid; else hi = mid - 1;
    }
    wb = lo;
    it_lo = a.item_off[lo]; it_hi = a.item_off[lo + 1];
    l_lo = a.list_off[lo]; l_hi = a.list_off[lo + 1];
  }
  // {bgj, first list position, number of queries}
  __device__ int4 describe(const AttnArgs &a, int qpi, int w) {
    while (w >= it_hi) {
      ++wb;
      it_lo = it_hi; it_hi = a.item_off[wb + 1];
      l_lo = l_hi; l_hi = a.list_off[wb + 1];
    }
    const int start = l_lo + (w - it_lo) * qpi;
    return make_int4(wb, start, min(qpi, l_hi - start), 0);
  }
};

template <int R, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    msa_prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = AttnCfg<R>;
  constexpr int QPI = C::QPI;
  // a K or V tile: BLK rows of 256 B as two 128B-swizzled halves (d 0..63,
  // 64..127) of BLK * 128 bytes each, in a 32 KB slot
  constexpr uint32_t kHalf = BLK * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t *ctl = smem + C::SMEM_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(ctl + C::CTL_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctl + C::CTL_MISC + 4);
  int4 *s_desc = reinterpret_cast<int4 *>(ctl + C::CTL_DESC);
  int4 *s_pre = reinterpret_cast<int4 *>(ctl + C::CTL_PRE);
  int *s_list = reinterpret_cast<int *>(ctl + C::CTL_LIST);
  auto bar = [&](int idx) { return bar0 + 8u * uint32_t(idx); };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::NQ; ++s) {
      mbar_init(bar(C::BAR_QFULL + s), 193);   // 192 copy completions + the list
      mbar_init(bar(C::BAR_STEMPTY + s), 4);   // the four softmax warps' stores
    }
    for (int x = 0; x < C::NKV; ++x) {
      mbar_init(bar(C::BAR_KVFULL + x), 1);
      mbar_init(bar(C::BAR_KVEMPTY + x), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(C::BAR_SFULL + u), 1);
      mbar_init(bar(C::BAR_PFULL + u), 128);
      mbar_init(bar(C::BAR_OFULL + u), 1);
      mbar_init(bar(C::BAR_TMEMPTY + u), 128);
    }
    mbar_init(bar(C::BAR_DRAIN), 1);
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

  const int n_bgj = a.q.B * a.G * a.nb;
  const int n_items = a.item_off[n_bgj];
  if (n_items > a.max_items && tid == 0) atomicCAS(a.status, 0, kStatusBadInput);
  // Each CTA takes a contiguous range of work items: consecutive items mostly
  // share their key block, whose K/V tiles are then loaded once.
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int w_begin = min(n_items, int(blockIdx.x) * per);
  const int n_loc = min(n_items, w_begin + per) - w_begin;

  if (warp < 8) {
    regs_dec_64();   // warpgroups 0 and 1, one instruction each
    if (warp == 0) {
      // ------------------------------------------------------ K/V producer
      if (lane == 0 && n_loc > 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        ItemWalk wk;
        wk.init(a, n_bgj, w_begin);
        int issued[C::NKV];
#pragma unroll
        for (int x = 0; x < C::NKV; ++x) issued[x] = -1;
        int prev = -1, m = -1;
        bool ok = true;
        for (int i = 0; i < n_loc && ok; ++i) {
          const int bgj = wk.describe(a, QPI, w_begin + i).x;
          if (bgj == prev) continue;
          prev = bgj;
          ++m;
          const int j = bgj % a.nb;
          const int g = (bgj / a.nb) % a.G;
          const int b = bgj / (a.nb * a.G);
#pragma unroll
          for (int h = 0; h < 2; ++h) {   // K of run m is tile sequence 2m, V is 2m+1
            const int tau = 2 * m + h;
            const int x = tau % C::NKV;
            if (!mbar_wait(bar(C::BAR_KVEMPTY + x), ((tau / C::NKV) & 1) ^ 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(C::BAR_KVFULL + x), 2 * kHalf);
            const uint32_t dst = s_base + C::SMEM_KV + x * kTile;
            // 4-D maps (d, G, key rows, sequences): the sequence's own map
            // (batch coordinate 0) or the launch's map over the batch
            const void *tm = a.kv_maps ? static_cast<const void *>(&a.kv_maps[2 * b + h])
                                       : (h ? static_cast<const void *>(&tm_v)
                                            : static_cast<const void *>(&tm_k));
            const int zb = a.kv_maps ? 0 : b;
            if (a.kv_maps) tensormap_acquire(tm);
            tma_load_4d(dst, tm, bar(C::BAR_KVFULL + x), 0, g, j * BLK, zb);
            tma_load_4d(dst + kHalf, tm, bar(C::BAR_KVFULL + x), 64, g, j * BLK, zb);
            issued[x] = tau;
          }
        }
        // let every load still in flight land before the CTA can exit
        for (int x = 0; x < C::NKV; ++x)
          if (issued[x] >= 0) mbar_wait_drain(bar(C::BAR_KVFULL + x), (issued[x] / C::NKV) & 1);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------ MMA issuer
      if (lane == 0 && n_loc > 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, BLK, 0, 0);
        constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
        int ns = 0, no = 0;          // next S and next O to issue (item indices)
        int m_s = -1, prev_bgj = -1; // run of item ns-1 and its key block
        // per in-flight item (ring of 4 by item index), 4 bits: the V tile of
        // its run (2), that tile's phase (1), whether the item opens its run (1)
        uint32_t ring = 0;
        bool q_seen = false, cur_new = false;
        int cur_bgj = -1;
        bool v_pending = false;      // O of a run's last-known item issued, successor unknown
        int v_tile = 0;              // ... and that run's V tile
        uint32_t idle = 0;
        uint64_t t_idle = 0;
        while (no < n_loc) {
          bool progressed = false;
          // ---- S_ns = Q K^T: needs the item's q rows, its K tile, a free TMEM slot
          if (ns < n_loc && ns < no + 2) {
            const int s = ns % C::NQ;
            if (!q_seen && mbar_test_wait(bar(C::BAR_QFULL + s), (ns / C::NQ) & 1)) {
              q_seen = true;
              cur_bgj = s_desc[s].x;
              cur_new = cur_bgj != prev_bgj;
            }
            if (q_seen) {
              const int m = cur_new ? m_s + 1 : m_s;
              const int xk = (2 * m) % C::NKV;
              const bool k_ok =
                  !cur_new || mbar_test_wait(bar(C::BAR_KVFULL + xk), ((2 * m) / C::NKV) & 1);
              if (k_ok && mbar_test_wait(bar(C::BAR_TMEMPTY + (ns & 1)), ((ns >> 1) & 1) ^ 1)) {
                tc_fence_after();
                fence_proxy_async_smem();   // cp.async-written q rows -> UMMA operand reads
                if (cur_new && ns > 0) {
                  // the previous run's last S is issued: its K tile frees when that completes
                  umma_commit(bar(C::BAR_KVEMPTY + (2 * m_s) % C::NKV));
                  if (v_pending) umma_commit(bar(C::BAR_KVEMPTY + v_tile));
                }
                v_pending = false;
                const uint32_t sq = s_base + C::SMEM_Q + s * kTile;
                const uint32_t sk = s_base + C::SMEM_KV + xk * kTile;
                const uint32_t d_tmem = tmem_base + (ns & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const int c = kk >> 2;
                  const uint32_t off = (kk & 3) * 32;
                  umma_f16_ss(d_tmem, sdesc_sw128(sq + c * 16384 + off, 16, 1024),
                              sdesc_sw128(sk + c * kHalf + off, 16, 1024), idesc_s, kk > 0);
                }
                umma_commit(bar(C::BAR_SFULL + (ns & 1)));
                {   // per in-flight item: V tile, its phase, whether the item opens a run
                  const int tv = 2 * m + 1;
                  const uint32_t e = uint32_t(tv % C::NKV) | (uint32_t((tv / C::NKV) & 1) << 2) |
                                     (cur_new ? 8u : 0u);
                  const uint32_t sh = 4u * uint32_t(ns & 3);
                  ring = (ring & ~(15u << sh)) | (e << sh);
                }
                m_s = m;
                prev_bgj = cur_bgj;
                q_seen = false;
                ++ns;
                progressed = true;
              }
            }
          }
          // ---- O_no = P V: needs the softmax's P and the item's V tile
          if (no < ns) {
            const uint32_t e = (ring >> (4u * uint32_t(no & 3))) & 15u;
            const int xv = int(e & 3u);
            const bool v_ok = !(e & 8u) || mbar_test_wait(bar(C::BAR_KVFULL + xv), (e >> 2) & 1u);
            if (v_ok && mbar_test_wait(bar(C::BAR_PFULL + (no & 1)), (no >> 1) & 1)) {
              tc_fence_after();
              // P (bf16 pairs over S's first BLK/2 columns) is A, from TMEM
              const uint32_t p_tmem = tmem_base + (no & 1) * 128;
              const uint32_t sv = s_base + C::SMEM_KV + xv * kTile;
              const uint32_t d_tmem = tmem_base + 256 + (no & 1) * 128;
#pragma unroll
              for (int kk = 0; kk < BLK / 16; ++kk)   // 16 keys (8 columns of P) each
                umma_f16_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(sv + kk * 2048, kHalf, 1024),
                            idesc_o, kk > 0);
              umma_commit(bar(C::BAR_OFULL + (no & 1)));
              // free run m's V tile once item no is known to be its last
              if (no + 1 < ns) {
                if ((ring >> (4u * uint32_t((no + 1) & 3))) & 8u)   // item no+1 opens a run
                  umma_commit(bar(C::BAR_KVEMPTY + xv));
              } else if (no + 1 < n_loc) {
                v_pending = true;
                v_tile = xv;
              }
              ++no;
              progressed = true;
            }
          }
          if (progressed) {
            idle = 0;
            t_idle = 0;
          } else {
            // back off between probes: a hot probe loop slows the shared
            // memory-instruction path of the warps sharing this SM sub-partition
            __nanosleep(32);
          }
          if (!progressed && (++idle & 255u) == 0) {
            if (*abort_flag) break;
            const uint64_t now = globaltimer_ns();
            if (t_idle == 0) {
              t_idle = now;
            } else if (now - t_idle > kWaitLimitNs) {
              *abort_flag = 1;
              atomicCAS(a.status, 0, kStatusTimeout);
              break;
            }
          }
        }
        // every UMMA issued has completed before TMEM can be released
        umma_commit(bar(C::BAR_DRAIN));
        mbar_wait_drain(bar(C::BAR_DRAIN), 0);
      }
    } else {
      // ------------------------------------------------------ q gather team
      // All six gather warps work on every item in turn: a warp's copy
      // issue rate is limited, so an item's 2048 16-byte copies are spread
      // over 192 threads (11 each).  Completion is signalled by the copies
      // themselves (cp.async.mbarrier.arrive.noinc), so the team moves on to
      // the next free stage while they land.
      const int gtid = tid - 64;             // 0..191
      const int wg = warp - 2;               // 0..5
      constexpr int kTeam = 192;
      constexpr int bar_id = 1;
      ItemWalk wk;
      // Every warp keeps the item's list entries in registers (entry 32c +
      // lane in ent[c]) and looks a query up with a shuffle.  The next
      // item's descriptor and entries are fetched while the copies land.
      constexpr int NE = (QPI + 31) / 32;
      int4 d = make_int4(0, 0, 0, 0);
      int ent[NE];
      auto load_entries = [&]() {
#pragma unroll
        for (int c = 0; c < NE; ++c)
          ent[c] = (32 * c + lane < d.z) ? a.list[d.y + 32 * c + lane] : 0;
      };
      if (gtid == 0 && n_loc > 0) {
        wk.init(a, n_bgj, w_begin);
        s_pre[0] = wk.describe(a, QPI, w_begin);
      }
      bar_sync_n(bar_id, kTeam);
      if (n_loc > 0) {
        d = s_pre[0];
        load_entries();
      }
      const int gran = lane & 15;
      for (int i = 0; i < n_loc; ++i) {
        const int s = i % C::NQ;
        bool ok = mbar_wait(bar(C::BAR_STEMPTY + s), ((i / C::NQ) & 1) ^ 1, abort_flag, a.status);
        if (!bar_and_n(bar_id, kTeam, ok)) break;
        if (gtid < 32) {   // publish the item: the MMA and the softmax read these
          if (gtid == 0) s_desc[s] = d;
#pragma unroll
          for (int c = 0; c < NE; ++c)
            if (32 * c + lane < d.z) s_list[s * QPI + 32 * c + lane] = ent[c];
          __syncwarp();
          if (gtid == 0) mbar_arrive(bar(C::BAR_QFULL + s));
        }
        const int bgj = d.x;
        const int g = (bgj / a.nb) % a.G;
        const int b = bgj / (a.nb * a.G);
        const uint16_t *qb = a.q_ptr + size_t(g) * R * kHeadDim + gran * 8;
        const int4 sq = qgeo_seq(a.q, b);
        const int qrow0 = sq.x - sq.y;        // + t: the query's packed row in q
        const uint32_t stq = s_base + C::SMEM_Q + s * kTile + (gran >> 3) * 16384;
        // row pair p = wg + 6*it (rows 2p, 2p+1): one coalesced 512-byte
        // copy per warp instruction
#pragma unroll
        for (int it = 0; it < 11; ++it) {
          const int p = wg + 6 * it;
          if (p < 64) {
            const int row = 2 * p + (lane >> 4);
            const int qi = row / R;
            const int hh = row % R;
            int e = ent[0];
#pragma unroll
            for (int c = 1; c < NE; ++c)
              if ((qi >> 5) == c) e = ent[c];   // warp-uniform: 2p, 2p+1 share qi >> 5
            const int t = __shfl_sync(0xffffffffu, e, qi & 31) >> 5;
            if (qi < d.z)
              cp_async16(stq + sw128_offset(row, gran & 7),
                         qb + (size_t(qrow0 + t) * a.H + hh) * kHeadDim);
          }
        }
        cp_async_arrive_noinc(bar(C::BAR_QFULL + s));
        if (gtid == 0 && i + 1 < n_loc) s_pre[0] = wk.describe(a, QPI, w_begin + i + 1);
        bar_sync_n(bar_id, kTeam);
        if (i + 1 < n_loc) {
          d = s_pre[0];
          load_entries();
        }
      }
    }
  } else {
    // -------------------------------------------------------- softmax + partials
    regs_inc_184();  // warpgroups 2 and 3, one instruction each
    const int u = (warp - 8) >> 2;         // even / odd items, TMEM slot u
    const int row = tid - 256 - 128 * u;   // TMEM lane = tile row
    const int bar_id = 4 + u;
    const uint32_t tm = tmem_base + u * 128 + (uint32_t((warp & 3) * 32) << 16);
    for (int i = u; i < n_loc; i += 2) {
      const int s = i % C::NQ;
      bool ok = mbar_wait(bar(C::BAR_QFULL + s), (i / C::NQ) & 1, abort_flag, a.status);
      if (!bar_and_n(bar_id, 128, ok)) break;
      const int4 d = s_desc[s];
      const int j = d.x % a.nb;
      const int qi = row / R;
      const bool valid = qi < d.z;
      const int t = valid ? (s_list[s * QPI + qi] >> 5) : 0;
      const int lim = valid ? (t - j * BLK) : (BLK - 1);   // last visible column
      ok = mbar_wait(bar(C::BAR_SFULL + u), (i >> 1) & 1, abort_flag, a.status);
      if (!bar_and_n(bar_id, 128, ok)) break;
      tc_fence_after();

      float v[BLK];
      {
        // every load is issued, then waited for, before any value is read
        float t0[32], t1[32], t2[32], t3[32];
        tmem_ld32(tm, t0);
        tmem_ld32(tm + 32, t1);
        if (BLK == 128) {
          tmem_ld32(tm + 64, t2);
          tmem_ld32(tm + 96, t3);
        }
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          v[x] = t0[x];
          v[32 + x] = t1[x];
          if (BLK == 128) {
            v[64 + x] = t2[x];
            v[96 + x] = t3[x];
          }
        }
      }
      // causal mask: only rows whose own block is j see fewer than BLK keys
      if (__any_sync(0xffffffffu, lim < BLK - 1)) {
#pragma unroll
        for (int x = 0; x < BLK; ++x) v[x] = (x <= lim) ? v[x] : -INFINITY;
      }
      float mc[BLK / 32];   // independent max chains, one per 32 columns
#pragma unroll
      for (int c4 = 0; c4 < BLK / 32; ++c4) mc[c4] = max3f(v[32 * c4], v[32 * c4 + 1], v[32 * c4 + 2]);
#pragma unroll
      for (int x = 3; x + 2 <= 31; x += 2) {
#pragma unroll
        for (int c4 = 0; c4 < BLK / 32; ++c4)
          mc[c4] = max3f(mc[c4], v[32 * c4 + x], v[32 * c4 + x + 1]);
      }
      float m = fmaxf(mc[0], v[31]);
#pragma unroll
      for (int c4 = 1; c4 < BLK / 32; ++c4) m = fmaxf(m, fmaxf(mc[c4], v[32 * c4 + 31]));
      const float mb = m * a.scale_log2;
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nmb2 = make_float2(-mb, -mb);
      float2 l2 = make_float2(0.f, 0.f);
      uint8_t *stage = smem + C::SMEM_Q + s * kTile;
      // P as bf16 pairs into S's own TMEM columns (S is all in registers):
      // 64 keys per 32 columns
#pragma unroll
      for (int h = 0; h < BLK / 64; ++h) {
        uint32_t pw[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = h * 64 + 2 * e;
          const float2 x = fma2(make_float2(v[c], v[c + 1]), sc2, nmb2);
          const float2 pp = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          l2 = add2(l2, pp);
          pw[e] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st32u(tm + h * 32, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::BAR_PFULL + u));

      ok = mbar_wait(bar(C::BAR_OFULL + u), (i >> 1) & 1, abort_flag, a.status);
      if (!bar_and_n(bar_id, 128, ok)) break;
      tc_fence_after();
      float ov[kHeadDim];   // the item's O row (all of d, whatever the block length)
      {
        float t0[32], t1[32], t2[32], t3[32];
        tmem_ld32(tm + 256, t0);
        tmem_ld32(tm + 288, t1);
        tmem_ld32(tm + 320, t2);
        tmem_ld32(tm + 352, t3);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          ov[x] = t0[x]; ov[32 + x] = t1[x]; ov[64 + x] = t2[x]; ov[96 + x] = t3[x];
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::BAR_TMEMPTY + u));   // slot u may take the next S

      // stage the normalised bf16 partial row (granule c at c ^ (row & 7))
      const float l = l2.x + l2.y;
      const float inv = 1.f / l;
      const float2 inv2 = make_float2(inv, inv);
      const int rho = d.y * R + row;       // partial row of (list position, head)
      uint8_t *orow = stage + row * 256;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float2 o0 = mul2(make_float2(ov[8 * c], ov[8 * c + 1]), inv2);
        const float2 o1 = mul2(make_float2(ov[8 * c + 2], ov[8 * c + 3]), inv2);
        const float2 o2 = mul2(make_float2(ov[8 * c + 4], ov[8 * c + 5]), inv2);
        const float2 o3 = mul2(make_float2(ov[8 * c + 6], ov[8 * c + 7]), inv2);
        const uint4 w = make_uint4(pack_bf16x2(o0.x, o0.y), pack_bf16x2(o1.x, o1.y),
                                   pack_bf16x2(o2.x, o2.y), pack_bf16x2(o3.x, o3.y));
        *reinterpret_cast<uint4 *>(orow + ((c ^ (rho & 7)) << 4)) = w;
      }
      if (valid) a.part_lse[rho] = m * a.scale + __logf(l);
      // each warp writes its own 32 rows (those holding a query) as soon as
      // they are staged
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int wrow0 = (warp & 3) * 32;
        const int nrows = min(32, d.z * R - wrow0);
        if (nrows > 0) {
          bulk_store(a.part_o + (size_t(d.y) * R + wrow0) * kHeadDim,
                     s_base + C::SMEM_Q + s * kTile + wrow0 * 256, uint32_t(nrows) * 256u);
          bulk_commit();
          bulk_wait_read_all();
        }
        mbar_arrive(bar(C::BAR_STEMPTY + s));   // with all four: the stage may take item i+3
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  cp_async_wait_all();   // nothing may still be landing in shared memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int R, int BLK>
cudaError_t launch_attn_r(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                          int num_sms, cudaStream_t st) {
  auto kern = msa_prefill_attn_kernel<R, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnCfg<R>::SMEM);
  if (e != cudaSuccess) return e;
  int grid = num_sms;
  if (a.max_items < grid) grid = a.max_items > 0 ? a.max_items : 1;
  kern<<<grid, kAttnThreads, AttnCfg<R>::SMEM, st>>>(tk, tv, a);
  return cudaGetLastError();
}

template <int BLK>
cudaError_t launch_attn_b(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                          int num_sms, cudaStream_t st) {
  switch (a.H / a.G) {
    case 1: return launch_attn_r<1, BLK>(tk, tv, a, num_sms, st);
    case 2: return launch_attn_r<2, BLK>(tk, tv, a, num_sms, st);
    case 4: return launch_attn_r<4, BLK>(tk, tv, a, num_sms, st);
    case 8: return launch_attn_r<8, BLK>(tk, tv, a, num_sms, st);
    case 16: return launch_attn_r<16, BLK>(tk, tv, a, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_prefill_attn(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                                int num_sms, cudaStream_t st) {
  return a.blk == 64 ? launch_attn_b<64>(tk, tv, a, num_sms, st)
                     : launch_attn_b<128>(tk, tv, a, num_sms, st);
}

// ---------------------------------------------------------------- combine
namespace {

// One warp per (packed row, h): merge the row's partials (normalised o_s,
// lse_s) into o = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M), M = max
// lse_s.  Slot s of the row lives at partial row rho_s = pos_of[g,row,s] * R
// + hh.  The selection row and the positions are loaded independently, then
// all of a lane's partial-row loads (4 of the d values of each slot, granule
// order undone) and its lse load are issued before any reduction.
template <int KCAP>
__global__ void __launch_bounds__(256) msa_combine_kernel(const CombineArgs a) {
  const long long wrow = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)a.Rc * a.H;
  if (wrow >= n_rows) return;
  const int h = (int)(wrow % a.H);
  const int rl = (int)(wrow / a.H);
  const int row = a.r0 + rl;
  const int b = qgeo_seq_of_row(a.q, row);
  const int4 sq = qgeo_seq(a.q, b);
  const int r = a.H / a.G;
  const int g = h / r;
  const int hh = h % r;
  const int32_t *sel = a.sel + ((long long)sq.w + (long long)g * a.q.sel_gs + (row - sq.x)) * a.top_k;
  const int32_t *pos = a.pos_of + ((long long)g * a.Rc + rl) * a.top_k;
  const bool in_k = lane < a.top_k;
  const int my_sel = in_k ? sel[lane] : -1;
  const int my_pos = in_k ? pos[lane] : 0;
  const bool mine = my_sel >= 0;
  const unsigned vmask = __ballot_sync(0xffffffffu, mine);
  const long long my_rho = mine ? (long long)my_pos * r + hh : 0;
  uint2 v[KCAP];
#pragma unroll
  for (int s = 0; s < KCAP; ++s) {
    v[s] = make_uint2(0u, 0u);
    const long long rho = __shfl_sync(0xffffffffu, my_rho, s);
    if ((vmask >> s) & 1u) {
      const int col = ((((lane >> 1) ^ int(rho & 7)) << 3) | ((lane & 1) << 2));
      v[s] = __ldcs(reinterpret_cast<const uint2 *>(a.part_o + rho * kHeadDim + col));
    }
  }
  const float my_lse = mine ? __ldcs(a.part_lse + my_rho) : -INFINITY;
  float M = my_lse;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (M > -INFINITY) {
    const float wmine = mine ? __expf(my_lse - M) : 0.f;
    wsum = wmine;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
#pragma unroll
    for (int s = 0; s < KCAP; ++s) {
      const float ws = __shfl_sync(0xffffffffu, wmine, s);
      acc[0] = fmaf(ws, bf16_lo(v[s].x), acc[0]);
      acc[1] = fmaf(ws, bf16_hi(v[s].x), acc[1]);
      acc[2] = fmaf(ws, bf16_lo(v[s].y), acc[2]);
      acc[3] = fmaf(ws, bf16_hi(v[s].y), acc[3]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint2 res;
  res.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  res.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  *reinterpret_cast<uint2 *>(a.out + ((size_t)row * a.H + h) * kHeadDim + lane * 4) = res;
  if (a.lse && lane == 0) a.lse[(size_t)row * a.H + h] = (wsum > 0.f) ? M + __logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
  const long long n_rows = (long long)a.Rc * a.H;
  if (n_rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n_rows + 7) / 8);
  if (a.top_k <= 4)
    msa_combine_kernel<4><<<grid, 256, 0, st>>>(a);
  else if (a.top_k <= 8)
    msa_combine_kernel<8><<<grid, 256, 0, st>>>(a);
  else if (a.top_k <= 16)
    msa_combine_kernel<16><<<grid, 256, 0, st>>>(a);
  else
    msa_combine_kernel<32><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
