// NSA-style branches beside MSA's selection ("MiniMax M3 sparse attention"
// explainer, mlqm.cn/news/533796, §3.1: DeepSeek NSA runs a compression, a
// selection and a sliding-window branch mixed by a learned gate; MSA keeps
// the selection alone).  The page names the other two branches without
// formulas; the readings implemented here:
//   window       query t attends its `window` most recent tokens, s in
//                [t-window+1, t], with exact softmax attention;
//   compression  block c is summarised by the mean of its keys and of its
//                values; query t attends the summaries of the blocks whose
//                every token lies at or before t (c <= (t+1)/block - 1); a
//                query with none gets a zero output;
//   gate         per (query, head) the caller gives three gate values, and
//                the output is g_cmp o_cmp + g_slc o_slc + g_win o_win.
//
// Kernels:
//   nsa_compress_kernel    block means of K and V (fp32 sums, bf16 out).
//   nsa_dense_attn_kernel  query-outer exact attention over a contiguous
//                visible key range per row: the window over the tokens, or
//                the completed blocks over the summaries.  One work item is
//                (b, g, 128/R consecutive queries x R heads), a 128-row tile
//                that one 4-D TMA box brings in.  The key tiles (128 keys)
//                that any row of the item sees are swept once: S = Q K^T in
//                TMEM, P = exp2(S - mr) as bf16 against a per-row reference
//                maximum mr, O += P V accumulated in TMEM across the tiles.
//                mr moves only when a tile raises the row's maximum by more
//                than 2^8 in P; the row's O columns and sum are then scaled
//                down in place (TMEM load, scale, TMEM store), which happens
//                a few times per row at most.
//   nsa_gate_kernel        the gate-weighted sum of the three branch outputs.
//
// Roles of nsa_dense_attn_kernel (one persistent CTA per SM, 12 warps):
//   warp 0     TMA producer: the item's Q tile, then K and V of each key
//              tile in turn, into a ring.
//   warp 1     TMEM owner and MMA issuer: S into two 128-column slots, O
//              into a third.  It issues S of tile i+1 before O of tile i,
//              so the softmax of the next tile overlaps P V.
//   warps 4-11 two softmax warpgroups, one row (TMEM lane) per thread each;
//              warpgroup h takes key columns 64h..64h+63 of every S tile
//              (and P's 16 KB half h, and d columns 64h.. of O).  The two
//              exchange each tile's row maxima through shared memory, so
//              both halves of a row use one reference, and their row sums
//              once at the end.
//   warps 2-3  idle.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kDenseThreads = 384;
constexpr int kDTile = 32768;                    // 128 rows x 256 B
constexpr int kDNkv = 3;                         // K/V ring depth
// shared memory (from a 1024-byte aligned base)
constexpr int kDSQ = 0;                          // Q tile
constexpr int kDSP = kDTile;                     // two P tiles
constexpr int kDSKV = 3 * kDTile;                // K/V ring
constexpr int kDCtl = kDSKV + kDNkv * kDTile;
// barrier slots
constexpr int kBQFull = 0, kBQEmpty = 1, kBKvFull = 2, kBKvEmpty = 2 + kDNkv,
              kBSFull = 2 + 2 * kDNkv, kBSEmpty = kBSFull + 2, kBPFull = kBSEmpty + 2,
              kBPEmpty = kBPFull + 2, kBOFull = kBPEmpty + 2, kBOEmpty = kBOFull + 1,
              kBDrain = kBOEmpty + 1, kDNumBars = kBDrain + 1;
constexpr int kDCtlMisc = kDNumBars * 8;         // tmem holder, abort flag
constexpr int kDCtlX = kDCtlMisc + 16;            // [2][128] row maxima, [2][128] row sums
constexpr int kDenseSmem = kDCtl + kDCtlX + 4 * 128 * 4 + 1024;
static_assert(kDenseSmem <= 232448, "shared memory budget");
// TMEM columns: S slots 0 and 128, O at 256 (512 allocated)
constexpr uint32_t kTmO = 256;

// Visible key range [lo, hi] of a query at position t (hi < lo: none).
__device__ __forceinline__ int dense_lo(const DenseAttnArgs &a, int t) {
  return a.mode == 0 ? max(0, t - a.window + 1) : 0;
}
__device__ __forceinline__ int dense_hi(const DenseAttnArgs &a, int t) {
  return a.mode == 0 ? t : (t + 1) / a.blk - 1;
}

struct DItem {
  int b, g, t0, kt_lo, n_kt;
};

// Work item u: query tiles from the last (the longest key ranges of the
// compression branch) to the first, every (b, g) of each.
__device__ __forceinline__ DItem dense_item(const DenseAttnArgs &a, int u, int qpi) {
  const int n_bg = a.B * a.G;
  const int qt = a.n_qt - 1 - u / n_bg;
  const int bg = u % n_bg;
  DItem w;
  w.b = bg / a.G;
  w.g = bg % a.G;
  w.t0 = qt * qpi;
  const int t_last = min(a.L - 1, w.t0 + qpi - 1);
  const int lo = dense_lo(a, w.t0), hi = dense_hi(a, t_last);
  if (hi < lo) {
    w.kt_lo = 0;
    w.n_kt = 0;
  } else {
    w.kt_lo = lo >> 7;
    w.n_kt = (hi >> 7) - w.kt_lo + 1;
  }
  return w;
}

// Item of this CTA in round r (snake order over the CTAs), or -1.
__device__ __forceinline__ int dense_round_item(int r, int n_items) {
  const int u = r * gridDim.x + ((r & 1) ? (gridDim.x - 1 - blockIdx.x) : blockIdx.x);
  return u < n_items ? u : -1;
}

template <int R>
__global__ void __launch_bounds__(kDenseThreads, 1)
    nsa_dense_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const DenseAttnArgs a) {
  constexpr int QPI = 128 / R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t *ctl = smem + kDCtl;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(ctl + kDCtlMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctl + kDCtlMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar(kBQFull), 1);
    mbar_init(bar(kBQEmpty), 1);
    for (int x = 0; x < kDNkv; ++x) {
      mbar_init(bar(kBKvFull + x), 1);
      mbar_init(bar(kBKvEmpty + x), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(kBSFull + u), 1);
      mbar_init(bar(kBSEmpty + u), 256);
      mbar_init(bar(kBPFull + u), 256);
      mbar_init(bar(kBPEmpty + u), 1);
    }
    mbar_init(bar(kBOFull), 1);
    mbar_init(bar(kBOEmpty), 256);
    mbar_init(bar(kBDrain), 1);
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
  const int n_items = a.B * a.G * a.n_qt;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int last[kDNkv];
#pragma unroll
      for (int x = 0; x < kDNkv; ++x) last[x] = -1;
      uint32_t kseq = 0;
      int qn = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = dense_round_item(r, n_items);
        if (u < 0) break;
        const DItem w = dense_item(a, u, QPI);
        if (w.n_kt == 0) continue;
        ok = mbar_wait(bar(kBQEmpty), (qn & 1) ^ 1, abort_flag, a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(kBQFull), kDTile);
        tma_load_4d(s_base + kDSQ, &tm_q, bar(kBQFull), 0, w.g * R, w.t0, w.b);
        tma_load_4d(s_base + kDSQ + 16384, &tm_q, bar(kBQFull), 64, w.g * R, w.t0, w.b);
        ++qn;
        // K and V of each tile in turn
        for (int step = 0; step < 2 * w.n_kt; ++step) {
          const int kt = step >> 1, is_v = step & 1;
          const int x = int(kseq % kDNkv);
          ok = mbar_wait(bar(kBKvEmpty + x), ((kseq / kDNkv) & 1) ^ 1, abort_flag, a.status);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(kBKvFull + x), kDTile);
          const void *tm = is_v ? static_cast<const void *>(&tm_v) : static_cast<const void *>(&tm_k);
          const uint32_t dst = s_base + kDSKV + x * kDTile;
          const int key0 = (w.kt_lo + kt) * 128;
          tma_load_4d(dst, tm, bar(kBKvFull + x), 0, w.g, key0, w.b);
          tma_load_4d(dst + 16384, tm, bar(kBKvFull + x), 64, w.g, key0, w.b);
          last[x] = int(kseq);
          ++kseq;
        }
      }
      // copies still in flight land before the CTA may exit
      for (int x = 0; x < kDNkv; ++x)
        if (last[x] >= 0) mbar_wait_drain(bar(kBKvFull + x), (uint32_t(last[x]) / kDNkv) & 1);
      if (qn > 0) mbar_wait_drain(bar(kBQFull), (qn - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t sq = s_base + kDSQ;
      uint32_t kseq = 0, scnt = 0, ocnt = 0;
      int item_n = 0;
      bool ok = true, issued = false;
      // S = Q K^T of the K tile with ring sequence number seq
      auto issue_s = [&](uint32_t seq) -> bool {
        const int x = int(seq % kDNkv);
        if (!mbar_wait(bar(kBKvFull + x), (seq / kDNkv) & 1, abort_flag, a.status)) return false;
        const int sl = int(scnt & 1);
        if (!mbar_wait(bar(kBSEmpty + sl), ((scnt >> 1) & 1) ^ 1, abort_flag, a.status))
          return false;
        tc_fence_after();
        const uint32_t sk = s_base + kDSKV + x * kDTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16_ss(tmem_base + sl * 128, sdesc_sw128(sq + off, 16, 1024),
                      sdesc_sw128(sk + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(bar(kBSFull + sl));
        umma_commit(bar(kBKvEmpty + x));   // the K tile is free once S completes
        issued = true;
        ++scnt;
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int u = dense_round_item(r, n_items);
        if (u < 0) break;
        const DItem w = dense_item(a, u, QPI);
        if (w.n_kt == 0) continue;
        ok = mbar_wait(bar(kBQFull), item_n & 1, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t p2 = kseq;   // K_kt at p2 + 2kt, V_kt at p2 + 2kt + 1
        ok = issue_s(p2);
        for (int kt = 0; kt < w.n_kt && ok; ++kt) {
          if (kt + 1 < w.n_kt) {
            ok = issue_s(p2 + 2 * (kt + 1));
            if (!ok) break;
          } else {
            umma_commit(bar(kBQEmpty));   // the item's last S is issued: Q frees on completion
          }
          const int pb = int(ocnt & 1);
          const uint32_t vseq = p2 + 2 * kt + 1;
          const int xv = int(vseq % kDNkv);
          ok = mbar_wait(bar(kBPFull + pb), (ocnt >> 1) & 1, abort_flag, a.status);
          if (ok) ok = mbar_wait(bar(kBKvFull + xv), (vseq / kDNkv) & 1, abort_flag, a.status);
          if (ok && kt == 0) ok = mbar_wait(bar(kBOEmpty), (item_n & 1) ^ 1, abort_flag, a.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sp = s_base + kDSP + pb * kDTile;
          const uint32_t sv = s_base + kDSKV + xv * kDTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // 16 keys per step, 64 per 16 KB half of P
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_f16_ss(tmem_base + kTmO, sdesc_sw128(sp + off, 16, 1024),
                        sdesc_sw128(sv + kk * 2048, 16384, 1024), idesc_o, (kt > 0 || kk > 0));
          }
          umma_commit(bar(kBPEmpty + pb));
          umma_commit(bar(kBKvEmpty + xv));
          ++ocnt;
        }
        if (!ok) break;
        umma_commit(bar(kBOFull));
        kseq = p2 + 2 * w.n_kt;
        ++item_n;
      }
      // every UMMA issued has completed before TMEM can be released
      if (issued) {
        umma_commit(bar(kBDrain));
        mbar_wait_drain(bar(kBDrain), 0);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax
    const int q4 = warp & 3;               // TMEM lane quadrant of this warp
    const int hc = (warp - 4) >> 2;        // key-column / d half of this warpgroup
    const int row = q4 * 32 + lane;        // tile row = TMEM lane
    const uint32_t tm_lane = tmem_base + (uint32_t(q4 * 32) << 16);
    const int qi = row / R, hh = row % R;
    float *x_max = reinterpret_cast<float *>(ctl + kDCtlX);   // [2][128]
    float *x_sum = x_max + 2 * 128;                             // [2][128]
    constexpr int bar_id = 1;
    uint32_t scnt = 0, pcnt = 0;
    int item_n = 0;
    bool ok = true;
    // this warpgroup's 64 columns of the next S slot (both loads issued,
    // then one wait)
    auto load_s = [&](float (&v)[64]) -> bool {
      const int sl = int(scnt & 1);
      bool w_ok = mbar_wait(bar(kBSFull + sl), (scnt >> 1) & 1, abort_flag, a.status);
      if (!bar_and_n(bar_id, 256, w_ok)) return false;
      tc_fence_after();
      float t0[32], t1[32];
      const uint32_t ta = tm_lane + sl * 128 + hc * 64;
      tmem_ld32(ta, t0);
      tmem_ld32(ta + 32, t1);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kBSEmpty + sl));
      ++scnt;
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        v[x] = t0[x];
        v[32 + x] = t1[x];
      }
      return true;
    };
    for (int r = 0; ok; ++r) {
      const int u = dense_round_item(r, n_items);
      if (u < 0) break;
      const DItem w = dense_item(a, u, QPI);
      const int t = w.t0 + qi;
      const bool valid = t < a.L;
      const int lo = valid ? dense_lo(a, t) : 1;
      const int hi = valid ? dense_hi(a, t) : 0;
      const size_t orow = (size_t(w.b) * a.L + t) * a.H + w.g * R + hh;
      if (w.n_kt == 0) {   // no row of the item sees a key: zero output
        if (valid) {
          uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * kHeadDim + hc * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          if (a.lse && hc == 0) a.lse[orow] = -INFINITY;
        }
        continue;
      }
      // ---- one sweep.  P is taken against a reference maximum mr that
      // moves only when a tile raises the row's maximum past mr by more
      // than 2^8 in P; then the row's O columns (in TMEM, after the last P V
      // has landed) and its sum are scaled down to the new reference.  So
      // P <= 2^8, and O is rescaled a few times per row at most.
      float mr = -INFINITY;   // reference maximum, raw score units
      float l = 0.f;
      for (int kt = 0; kt < w.n_kt; ++kt) {
        float v[64];
        ok = load_s(v);
        if (!ok) break;
        const int c0 = lo - (w.kt_lo + kt) * 128 - hc * 64, c1 = hi - (w.kt_lo + kt) * 128 - hc * 64;
        float tmx = -INFINITY;
#pragma unroll
        for (int x = 0; x < 64; ++x) tmx = (x >= c0 && x <= c1) ? fmaxf(tmx, v[x]) : tmx;
        x_max[hc * 128 + row] = tmx;   // both halves of the row share the reference
        bar_sync_n(bar_id, 256);
        tmx = fmaxf(tmx, x_max[(hc ^ 1) * 128 + row]);
        const bool resc =
            tmx > -INFINITY && (mr == -INFINITY || (tmx - mr) * a.scale_log2 > 8.f);
        const float alpha =
            resc ? (mr == -INFINITY ? 0.f : fast_exp2((mr - tmx) * a.scale_log2)) : 1.f;
        l *= alpha;
        if (kt > 0 && __any_sync(0xffffffffu, resc && mr > -INFINITY)) {
          // O holds the earlier tiles of this warp's rows: wait for the last
          // P V, then scale this warpgroup's 64 columns in place
          const uint32_t u = pcnt - 1;
          bool r_ok = mbar_wait(bar(kBPEmpty + (u & 1)), (u >> 1) & 1, abort_flag, a.status);
          if (__all_sync(0xffffffffu, r_ok)) {
            tc_fence_after();
#pragma unroll 1
            for (int c32 = 0; c32 < 2; ++c32) {   // 32 columns at a time: few live registers
              float t0[32];
              const uint32_t to = tm_lane + kTmO + hc * 64 + c32 * 32;
              tmem_ld32(to, t0);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) t0[x] *= alpha;
              tmem_st32(to, t0);
              tmem_wait_st();
            }
            tc_fence_before();
          } else {
            ok = false;
          }
        }
        if (resc) mr = tmx;
        const float mb = (mr == -INFINITY) ? 0.f : mr * a.scale_log2;
        const int pb = int(pcnt & 1);
        bool w_ok = ok && mbar_wait(bar(kBPEmpty + pb), ((pcnt >> 1) & 1) ^ 1, abort_flag, a.status);
        if (!bar_and_n(bar_id, 256, w_ok)) {
          ok = false;
          break;
        }
        uint8_t *stile = smem + kDSP + pb * kDTile + hc * 16384;
#pragma unroll
        for (int gb = 0; gb < 8; ++gb) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = gb * 8 + e * 2;
            const float p0 =
                (c >= c0 && c <= c1) ? fast_exp2(fmaf(v[c], a.scale_log2, -mb)) : 0.f;
            const float p1 =
                (c + 1 >= c0 && c + 1 <= c1) ? fast_exp2(fmaf(v[c + 1], a.scale_log2, -mb)) : 0.f;
            l += p0 + p1;
            w4[e] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4 *>(stile + sw128_offset(row, gb)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(kBPFull + pb));
        ++pcnt;
      }
      if (!ok) break;
      x_sum[hc * 128 + row] = l;
      // ---- O / l
      bool w_ok = mbar_wait(bar(kBOFull), item_n & 1, abort_flag, a.status);
      if (!bar_and_n(bar_id, 256, w_ok)) break;   // also publishes the partial sums
      l += x_sum[(hc ^ 1) * 128 + row];
      tc_fence_after();
      float o[64];
      {
        float t0[32], t1[32];
        tmem_ld32(tm_lane + kTmO + hc * 64, t0);
        tmem_ld32(tm_lane + kTmO + hc * 64 + 32, t1);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          o[x] = t0[x];
          o[32 + x] = t1[x];
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBOEmpty));
      ++item_n;
      if (valid) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * kHeadDim + hc * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c] = make_uint4(pack_bf16x2(o[8 * c] * inv, o[8 * c + 1] * inv),
                              pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv),
                              pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv),
                              pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv));
        if (a.lse && hc == 0) a.lse[orow] = l > 0.f ? mr * a.scale + __logf(l) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// k_cmp[b, c, g, :] = mean of k[b, s, g, :] over the rows s < L of block c,
// and the same for v.  One warp per (b, c, g, tensor); lane i sums dims
// 4i..4i+3 in fp32.
__global__ void __launch_bounds__(256)
    nsa_compress_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
                        uint16_t *__restrict__ k_cmp, uint16_t *__restrict__ v_cmp, int B, int L,
                        int G, int blk, int nbc) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long n = (long long)B * nbc * G * 2;
  if (w >= n) return;
  const int which = int(w & 1);
  long long rest = w >> 1;
  const int g = int(rest % G);
  rest /= G;
  const int c = int(rest % nbc);
  const int b = int(rest / nbc);
  const uint16_t *src = which ? v : k;
  const int s0 = c * blk, s1 = min(L, s0 + blk);
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 8
  for (int s = s0; s < s1; ++s) {
    const uint2 x =
        __ldcs(reinterpret_cast<const uint2 *>(src + ((size_t(b) * L + s) * G + g) * kHeadDim) + lane);
    acc0 += bf16_lo(x.x);
    acc1 += bf16_hi(x.x);
    acc2 += bf16_lo(x.y);
    acc3 += bf16_hi(x.y);
  }
  const float inv = 1.f / float(s1 - s0);
  uint16_t *dst = (which ? v_cmp : k_cmp) + ((size_t(b) * nbc + c) * G + g) * kHeadDim;
  reinterpret_cast<uint2 *>(dst)[lane] =
      make_uint2(pack_bf16x2(acc0 * inv, acc1 * inv), pack_bf16x2(acc2 * inv, acc3 * inv));
}

// out[r, :] = g_cmp o_cmp[r, :] + g_slc o_slc[r, :] + g_win o_win[r, :] for
// the rows r = (b*L + t)*H + h; 16 threads per row, 8 values each.  out may
// be one of the inputs (each thread reads its values before writing them).
__global__ void __launch_bounds__(256)
    nsa_gate_kernel(const float *__restrict__ gates, const uint16_t *o_cmp, const uint16_t *o_slc,
                    const uint16_t *o_win, uint16_t *out, long long rows) {
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  const long long r = i >> 4;
  if (r >= rows) return;
  const int c = int(i & 15);
  const float g0 = gates[3 * r], g1 = gates[3 * r + 1], g2 = gates[3 * r + 2];
  const size_t e = size_t(r) * kHeadDim + c * 8;
  const uint4 x = *reinterpret_cast<const uint4 *>(o_cmp + e);
  const uint4 y = *reinterpret_cast<const uint4 *>(o_slc + e);
  const uint4 z = *reinterpret_cast<const uint4 *>(o_win + e);
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w},
                 zs[4] = {z.x, z.y, z.z, z.w};
  uint32_t res[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = g0 * bf16_lo(xs[j]) + g1 * bf16_lo(ys[j]) + g2 * bf16_lo(zs[j]);
    const float hi = g0 * bf16_hi(xs[j]) + g1 * bf16_hi(ys[j]) + g2 * bf16_hi(zs[j]);
    res[j] = pack_bf16x2(lo, hi);
  }
  *reinterpret_cast<uint4 *>(out + e) = make_uint4(res[0], res[1], res[2], res[3]);
}

template <int R>
cudaError_t launch_dense_r(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           const DenseAttnArgs &a, int num_sms, cudaStream_t st) {
  auto kern = nsa_dense_attn_kernel<R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDenseSmem);
  if (e != cudaSuccess) return e;
  const int n_items = a.B * a.G * a.n_qt;
  const int grid = n_items < num_sms ? n_items : num_sms;
  kern<<<grid, kDenseThreads, kDenseSmem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dense_attn(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                              const DenseAttnArgs &a, int num_sms, cudaStream_t st) {
  if ((long long)a.B * a.G * a.n_qt == 0) return cudaSuccess;
  switch (a.H / a.G) {
    case 1: return launch_dense_r<1>(tq, tk, tv, a, num_sms, st);
    case 2: return launch_dense_r<2>(tq, tk, tv, a, num_sms, st);
    case 4: return launch_dense_r<4>(tq, tk, tv, a, num_sms, st);
    case 8: return launch_dense_r<8>(tq, tk, tv, a, num_sms, st);
    case 16: return launch_dense_r<16>(tq, tk, tv, a, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_nsa_compress(const uint16_t *k, const uint16_t *v, uint16_t *k_cmp,
                                uint16_t *v_cmp, int B, int L, int G, int blk, cudaStream_t st) {
  const int nbc = (L + blk - 1) / blk;
  const long long warps = (long long)B * nbc * G * 2;
  if (warps == 0) return cudaSuccess;
  nsa_compress_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(k, v, k_cmp, v_cmp, B, L, G,
                                                                   blk, nbc);
  return cudaGetLastError();
}

cudaError_t launch_nsa_gate(const float *gates, const uint16_t *o_cmp, const uint16_t *o_slc,
                            const uint16_t *o_win, uint16_t *out, long long rows, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  nsa_gate_kernel<<<(unsigned)((rows * 16 + 255) / 256), 256, 0, st>>>(gates, o_cmp, o_slc, o_win,
                                                                       out, rows);
  return cudaGetLastError();
}

}  // namespace msa
