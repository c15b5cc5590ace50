// Main Branch, backward pass: gradients of the exact attention over the
// selected blocks with respect to q, k and v, the selection held fixed.
// researchpapers.dev "MiniMax Sparse Attention", section "机制" (training
// paragraph): the index branch learns from a KL loss against the main
// branch and its path into the main attention carries no gradient, so the
// main branch's backward is that of ordinary softmax attention restricted to
// the selected tokens.  For one (query t, head h) row with probabilities P
// over its tokens s (P = exp(scale q.k_s - lse), lse from the forward):
//   dP_s = do . v_s,   D = do . o,   dZ_s = P_s (dP_s - D)
//   dq  = scale sum_s dZ_s k_s,  dk_s += scale dZ_s q,  dv_s += P_s do.
//
// Organised key-block-outer, on the forward's reverse index: one unit =
// one (b, g, key block j) with every (query, slot) that selected j, taken
// whole by one CTA so that dK_j and dV_j accumulate in TMEM and are written
// once, without atomics.  The key tile is 128 rows: a 128-token block fills
// it, a 64-token block fills its first half (the other keys are masked out
// of P and dZ, so their dK/dV rows stay zero and are not written), and the
// block that holds a sequence's last key loads zeros past it.  A unit's queries are processed as 128-row items
// (128/R queries x R heads), as in the forward:
//   gather   q and do rows of the item (cp.async, 128B-swizzled K-major)
//   S  = Q K_j^T, dP = dO V_j^T          (UMMA, fp32 in TMEM cols 0-255)
//   softmax  P and dZ as bf16 into shared memory (rows x keys, K-major)
//   dV_j += P^T dO, dK_j += dZ^T Q       (UMMA, A operand MN-major: the
//                                         same tiles read transposed)
//   dQ_part = dZ K_j                     (UMMA into TMEM cols 0-127)
//   dQ_part * scale -> bf16 partial row of (list position, head)
// and after the unit's last item dK_j (* scale) and dV_j leave as bf16.  A
// second kernel sums each query row's <= top_k partials into dq.  Long
// inputs run in query chunks, each with its own reverse index; dK/dV are
// then carried across chunks in fp32 accumulators (read, added to and
// rewritten by the one CTA that owns the block) and the last chunk writes
// them as bf16.  The next
// item's gather starts as soon as the dV/dK products have read the q/do
// tiles (the dQ product has its own commit), and the next unit's K/V loads
// as soon as the dQ product has read K; both overlap the epilogues.  The dQ
// partial rows are staged in the P tile and leave by bulk copy.  Units are handed out by an atomic counter, low key blocks
// (the longest lists) first.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kTileB = 32768;                 // 128 rows x 256 B
// shared memory (from a 1024-byte aligned base)
constexpr int kSK = 0, kSV = kTileB, kSQ = 2 * kTileB, kSDO = 3 * kTileB, kSP = 4 * kTileB,
              kSDZ = 5 * kTileB, kSCtl = 6 * kTileB;
constexpr int kBarKv = 0, kBarQ = 1, kBarMma = 2, kBarDrain = 3, kBarDq = 4;
constexpr int kCtlHolder = 32, kCtlAbort = 36, kCtlUnit = 40;
constexpr int kBwdSmem = kSCtl + 64 + 1024;
static_assert(kBwdSmem <= 232448, "shared memory budget");

// TMEM columns: S / dQ, dP, dV, dK (128 lanes x 128 fp32 each).
constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDV = 256, kTmDK = 384;

// 32 consecutive dk or dv values of one row (element offset e0): x * f for
// this query chunk (x null: nothing from this chunk).  A single-chunk call
// writes them as bf16.  With several chunks they are added to the fp32
// accumulator (zeroed before the first chunk), and the last chunk writes
// the sum as bf16.
__device__ __forceinline__ void put_grad32(const float *x, float f, size_t e0, uint16_t *out,
                                           float *acc, bool last) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = x ? x[i] * f : 0.f;
  if (acc) {
    const float4 *src = reinterpret_cast<const float4 *>(acc + e0);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 w = src[c];
      v[4 * c] += w.x; v[4 * c + 1] += w.y; v[4 * c + 2] += w.z; v[4 * c + 3] += w.w;
    }
  }
  if (!acc || last) {
    uint4 *dst = reinterpret_cast<uint4 *>(out + e0);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      dst[c] = make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                          pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                          pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
  } else {
    float4 *dst = reinterpret_cast<float4 *>(acc + e0);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}

// One (b, g, key block j) unit: its reverse-index list [l_lo, l_lo + n_q).
struct Unit {
  int bgj, b, g, j, l_lo, n_q;
};

template <int R, int BLK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    msa_backward_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const BwdArgs a) {
  constexpr int QPI = 128 / R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t *ctl = smem + kSCtl;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(ctl + kCtlHolder);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctl + kCtlAbort);
  volatile int *s_unit = reinterpret_cast<volatile int *>(ctl + kCtlUnit);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row = tid & 127;        // tile row (TMEM lane) of this thread
  const int half = tid >> 7;        // which 64 of the 128 columns it handles

  if (tid == 0) {
    mbar_init(bar(kBarKv), 1);
    mbar_init(bar(kBarQ), kBwdThreads);   // one cp.async completion per thread
    mbar_init(bar(kBarMma), 1);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarDq), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  // padding rows of a partial item, and with 64-key blocks key rows 64..127
  // of the K/V tiles, keep whatever the buffers held; start from zeros so
  // that they are finite (their P and dZ are 0)
  for (int x = tid; x < 4 * kTileB / 16; x += kBwdThreads)
    reinterpret_cast<uint4 *>(smem + kSK)[x] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tm_row = tmem_base + (uint32_t((warp & 3) * 32) << 16);

  const int n_bg = a.B * a.G;
  const int n_units = n_bg * a.nb;
  const float log2e = 1.4426950408889634f;

  // Next unit with at least one query (all threads).  Units nobody selected
  // get zero gradients here.
  auto fetch_unit = [&](Unit &un) -> bool {
    for (;;) {
      if (tid == 0) *s_unit = atomicAdd(a.unit_ctr, 1);
      __syncthreads();
      const int u = *s_unit;
      __syncthreads();
      if (u >= n_units) return false;
      un.j = u / n_bg;
      const int bg = u % n_bg;
      un.b = bg / a.G;
      un.g = bg % a.G;
      un.bgj = bg * a.nb + un.j;
      un.l_lo = a.list_off[un.bgj];
      un.n_q = a.list_off[un.bgj + 1] - un.l_lo;
      if (un.n_q > 0) return true;
      if (a.acc_dk && !a.last) continue;   // an earlier or later chunk writes this block
      const int key = un.j * BLK + row;
      if (row < BLK && key < a.L) {
        const size_t r0 = ((size_t(un.b) * a.L + key) * a.G + un.g) * kHeadDim + half * 64;
        put_grad32(nullptr, 0.f, r0, a.dk, a.acc_dk, a.last);
        put_grad32(nullptr, 0.f, r0 + 32, a.dk, a.acc_dk, a.last);
        put_grad32(nullptr, 0.f, r0, a.dv, a.acc_dv, a.last);
        put_grad32(nullptr, 0.f, r0 + 32, a.dv, a.acc_dv, a.last);
      }
    }
  };
  // K_j and V_j of a unit into their tiles (thread 0): BLK key rows, the
  // maps' row extent ending at the sequence's last key (rows past it load
  // as zeros)
  auto load_kv = [&](const Unit &un) {
    const int z = un.j * BLK;
    mbar_arrive_expect_tx(bar(kBarKv), 4u * BLK * 128u);
    tma_load_4d(s_base + kSK, &tm_k, bar(kBarKv), 0, un.g, z, un.b);
    tma_load_4d(s_base + kSK + 16384, &tm_k, bar(kBarKv), 64, un.g, z, un.b);
    tma_load_4d(s_base + kSV, &tm_v, bar(kBarKv), 0, un.g, z, un.b);
    tma_load_4d(s_base + kSV + 16384, &tm_v, bar(kBarKv), 64, un.g, z, un.b);
  };
  // Query positions of this thread's eight gather rows of item `it` of a
  // unit (-1 past the item's end): row pairs p = warp + 8 i (rows 2p, 2p+1).
  auto gather_rows = [&](const Unit &un, int it, int (&tq)[8]) {
    const int start = un.l_lo + it * QPI;
    const int n = min(QPI, un.n_q - it * QPI);
#pragma unroll
    for (int i = 0; i < 8; ++i) {   // all loads first: one memory latency
      const int qi = (2 * (warp + 8 * i) + (lane >> 4)) / R;
      tq[i] = qi < n ? (a.list[start + qi] >> 5) : -1;
    }
  };
  // q and do rows of a unit's item (all threads), one 512-byte copy per warp
  // instruction, given the rows' query positions
  auto gather = [&](const Unit &un, const int (&tq)[8]) {
    const int gran = lane & 15;
    const uint32_t off_g = (gran >> 3) * 16384;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 2 * (warp + 8 * i) + (lane >> 4);
      if (tq[i] >= 0) {
        const size_t src =
            ((size_t(un.b) * a.L + tq[i]) * a.H + un.g * R + r % R) * kHeadDim + gran * 8;
        const uint32_t dst = off_g + sw128_offset(r, gran & 7);
        cp_async16(s_base + kSQ + dst, a.q + src);
        cp_async16(s_base + kSDO + dst, a.dout + src);
      }
    }
    cp_async_arrive_noinc(bar(kBarQ));
  };

  Unit cur;
  bool have = fetch_unit(cur);
  bool kv_inflight = false, mma_issued = false;   // (thread 0)
  if (have) {
    if (tid == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      load_kv(cur);
      kv_inflight = true;
    }
    int tq0[8];
    gather_rows(cur, 0, tq0);
    gather(cur, tq0);
  }
  int it = 0;          // item of the current unit
  uint32_t n_items = 0, n_units_done = 0;
  bool ok = true;

  while (have) {
    const int start = cur.l_lo + it * QPI;
    const int n = min(QPI, cur.n_q - it * QPI);
    // this thread's row: query, head, lse and D
    const int qi = row / R;
    const bool valid = qi < n;
    int lim = -1;              // last visible key column of the row (-1: none)
    float lse2 = 0.f, dlt = 0.f;
    if (valid) {
      const int t = a.list[start + qi] >> 5;
      const size_t ri = (size_t(cur.b) * a.L + t) * a.H + cur.g * R + row % R;
      lse2 = a.lse[ri] * log2e;
      dlt = a.delta[ri];
      lim = min(BLK - 1, t - cur.j * BLK);
    }
    // the next item's gather rows, when it belongs to this unit: loaded now,
    // their latency hides behind this item's products
    int tq_next[8];
    const bool next_in_unit = (it + 1) * QPI < cur.n_q;
    if (next_in_unit) gather_rows(cur, it + 1, tq_next);
    // ---- S = Q K^T, dP = dO V^T
    ok = mbar_wait(bar(kBarQ), n_items & 1, abort_flag, a.status);
    if (ok && it == 0) ok = mbar_wait(bar(kBarKv), n_units_done & 1, abort_flag, a.status);
    if (!__syncthreads_and(ok)) break;
    if (tid == 0) {
      kv_inflight = false;
      mma_issued = true;
      tc_fence_after();
      fence_proxy_async_smem();   // cp.async-written rows -> UMMA operand reads
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_f16_ss(tmem_base + kTmS, sdesc_sw128(s_base + kSQ + off, 16, 1024),
                    sdesc_sw128(s_base + kSK + off, 16, 1024), idesc, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_f16_ss(tmem_base + kTmDP, sdesc_sw128(s_base + kSDO + off, 16, 1024),
                    sdesc_sw128(s_base + kSV + off, 16, 1024), idesc, kk > 0);
      }
      umma_commit(bar(kBarMma));
    }
    ok = mbar_wait(bar(kBarMma), 0, abort_flag, a.status);
    if (lane == 0 && half == 0) bulk_wait_read_all();   // the last item's staged dq rows
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // ---- P and dZ (bf16, key columns half*64 .. +64 of this row)
    {
      float s0[32], s1[32], d0[32], d1[32];
      tmem_ld32(tm_row + kTmS + half * 64, s0);
      tmem_ld32(tm_row + kTmS + half * 64 + 32, s1);
      tmem_ld32(tm_row + kTmDP + half * 64, d0);
      tmem_ld32(tm_row + kTmDP + half * 64 + 32, d1);
      tmem_wait_ld();
      uint8_t *sp = smem + kSP + half * 16384;
      uint8_t *sz = smem + kSDZ + half * 16384;
#pragma unroll
      for (int gb = 0; gb < 8; ++gb) {
        uint32_t wp[4], wz[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float p2[2], z2[2];
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int c = gb * 8 + e * 2 + w;        // 0..63 within this half
            const float sv = c < 32 ? s0[c] : s1[c - 32];
            const float dv = c < 32 ? d0[c] : d1[c - 32];
            const float pv = (half * 64 + c <= lim) ? fast_exp2(fmaf(sv, a.scale_log2, -lse2)) : 0.f;
            p2[w] = pv;
            z2[w] = pv * (dv - dlt);
          }
          wp[e] = pack_bf16x2(p2[0], p2[1]);
          wz[e] = pack_bf16x2(z2[0], z2[1]);
        }
        *reinterpret_cast<uint4 *>(sp + sw128_offset(row, gb)) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
        *reinterpret_cast<uint4 *>(sz + sw128_offset(row, gb)) = make_uint4(wz[0], wz[1], wz[2], wz[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- dV += P^T dO, dK += dZ^T Q, dQ = dZ K
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, 128, 1, 1);
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, 128, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {   // K = 16 tile rows per step
        const uint32_t off = kk * 2048;
        umma_f16_ss(tmem_base + kTmDV, sdesc_sw128(s_base + kSP + off, 16384, 1024),
                    sdesc_sw128(s_base + kSDO + off, 16384, 1024), idesc_t, (it > 0 || kk > 0));
        umma_f16_ss(tmem_base + kTmDK, sdesc_sw128(s_base + kSDZ + off, 16384, 1024),
                    sdesc_sw128(s_base + kSQ + off, 16384, 1024), idesc_t, (it > 0 || kk > 0));
      }
      umma_commit(bar(kBarMma));   // the q/do tiles are free once these complete
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {   // K = 16 keys per step
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_f16_ss(tmem_base + kTmS, sdesc_sw128(s_base + kSDZ + off, 16, 1024),
                    sdesc_sw128(s_base + kSK + kk * 2048, 16384, 1024), idesc_q, kk > 0);
      }
      umma_commit(bar(kBarDq));
    }
    ok = mbar_wait(bar(kBarMma), 1, abort_flag, a.status);
    if (!__syncthreads_and(ok)) break;
    ++n_items;
    // ---- the q/do tiles are free: start the next item's copies while the
    // dQ product and the epilogues run
    const bool unit_end = !next_in_unit;
    Unit nxt = cur;
    bool have_next = true;
    if (unit_end) have_next = fetch_unit(nxt);
    if (have_next) {
      if (unit_end) gather_rows(nxt, 0, tq_next);
      gather(nxt, tq_next);
    }
    ok = mbar_wait(bar(kBarDq), (n_items - 1) & 1, abort_flag, a.status);
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // the K/V tiles (read by the dQ product) are free at a unit's end
    if (unit_end && have_next && tid == 0) {
      load_kv(nxt);
      kv_inflight = true;
    }
    // ---- dQ partial rows: (list position start + qi, head hh) -> partial
    // row rho = start*R + r, bf16, its 16-byte granule c at c ^ (rho & 7);
    // staged in the P tile (free now) and written with one bulk copy per
    // 32 rows
    {
      float q0[32], q1[32];
      tmem_ld32(tm_row + kTmS + half * 64, q0);
      tmem_ld32(tm_row + kTmS + half * 64 + 32, q1);
      tmem_wait_ld();
      const int rho7 = (start * R + row) & 7;
      uint8_t *srow = smem + kSP + row * 256;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float *x = c < 4 ? q0 + 8 * c : q1 + 8 * (c - 4);
        const uint4 w = make_uint4(pack_bf16x2(x[0] * a.scale, x[1] * a.scale),
                                   pack_bf16x2(x[2] * a.scale, x[3] * a.scale),
                                   pack_bf16x2(x[4] * a.scale, x[5] * a.scale),
                                   pack_bf16x2(x[6] * a.scale, x[7] * a.scale));
        *reinterpret_cast<uint4 *>(srow + ((half * 8 + (c ^ rho7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      __syncthreads();   // both halves of each row staged
      if (half == 0 && lane == 0) {
        const int wrow0 = warp * 32;
        const int nrows = min(32, n * R - wrow0);
        if (nrows > 0) {
          bulk_store(a.part_dq + (size_t(start) * R + wrow0) * kHeadDim,
                     s_base + kSP + wrow0 * 256, uint32_t(nrows) * 256u);
          bulk_commit();
        }
      }
    }
    // ---- unit end: dK_j (* scale) and dV_j rows (key = TMEM lane) as bf16
    if (unit_end) {
      const int key = cur.j * BLK + row;
      const bool own = row < BLK && key < a.L;   // TMEM lanes of this block's keys
      const size_t r0 = ((size_t(cur.b) * a.L + key) * a.G + cur.g) * kHeadDim + half * 64;
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        float x0[32], x1[32];   // (the loads are warp-wide: every lane takes part)
        tmem_ld32(tm_row + (m ? kTmDK : kTmDV) + half * 64, x0);
        tmem_ld32(tm_row + (m ? kTmDK : kTmDV) + half * 64 + 32, x1);
        tmem_wait_ld();
        if (!own) continue;
        const float f = m ? a.scale : 1.f;
        uint16_t *out = m ? a.dk : a.dv;
        float *acc = m ? a.acc_dk : a.acc_dv;
        put_grad32(x0, f, r0, out, acc, a.last);
        put_grad32(x1, f, r0 + 32, out, acc, a.last);
      }
      ++n_units_done;
    }
    tc_fence_before();
    __syncthreads();   // TMEM read out before the next item's UMMAs overwrite it
    if (!have_next) break;
    it = unit_end ? 0 : it + 1;
    cur = nxt;
  }

  // nothing may still be landing in shared memory or running on the tensor
  // cores when the CTA releases them
  cp_async_wait_all();
  if (lane == 0 && half == 0) bulk_wait_all();
  if (tid == 0) {
    if (kv_inflight) mbar_wait_drain(bar(kBarKv), n_units_done & 1);
    if (mma_issued) {
      umma_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// D[b,t,h] = do . o (fp32), one warp per row.
__global__ void __launch_bounds__(256) bwd_delta_kernel(const uint16_t *__restrict__ o,
                                                        const uint16_t *__restrict__ dout,
                                                        float *__restrict__ delta, long long rows) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const uint2 x = __ldcs(reinterpret_cast<const uint2 *>(o + w * kHeadDim) + lane);
  const uint2 y = __ldcs(reinterpret_cast<const uint2 *>(dout + w * kHeadDim) + lane);
  float s = bf16_lo(x.x) * bf16_lo(y.x);
  s = fmaf(bf16_hi(x.x), bf16_hi(y.x), s);
  s = fmaf(bf16_lo(x.y), bf16_lo(y.y), s);
  s = fmaf(bf16_hi(x.y), bf16_hi(y.y), s);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) delta[w] = s;
}

// dq[b,t,h] = sum over the row's selected slots of its fp32 partial rows
// (already scaled), one warp per (b, t, h), four columns per lane.
template <int KCAP>
__global__ void __launch_bounds__(256) bwd_dq_reduce_kernel(const BwdArgs a) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)a.Rc * a.H;   // the chunk's rows
  if (w >= n_rows) return;
  const int h = (int)(w % a.H);
  const int rl = (int)(w / a.H);
  const int row = a.r0 + rl;              // packed row b*L + t
  const int b = row / a.L, t = row % a.L;
  const int r = a.H / a.G;
  const int g = h / r, hh = h % r;
  const size_t es = ((size_t(b) * a.G + g) * a.L + t) * a.top_k;     // sel row
  const size_t ep = (size_t(g) * a.Rc + rl) * a.top_k;               // pos_of row (chunk)
  const bool in_k = lane < a.top_k;
  const int my_sel = in_k ? a.sel[es + lane] : -1;
  const long long my_rho = (my_sel >= 0) ? (long long)a.pos_of[ep + lane] * r + hh : -1;
  uint2 v[KCAP];
#pragma unroll
  for (int s = 0; s < KCAP; ++s) {
    const long long rho = __shfl_sync(0xffffffffu, my_rho, s);
    v[s] = make_uint2(0u, 0u);
    if (rho >= 0) {
      const int col = (((lane >> 1) ^ int(rho & 7)) << 3) | ((lane & 1) << 2);
      v[s] = __ldcs(reinterpret_cast<const uint2 *>(a.part_dq + rho * kHeadDim + col));
    }
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < KCAP; ++s) {
    acc.x += bf16_lo(v[s].x); acc.y += bf16_hi(v[s].x);
    acc.z += bf16_lo(v[s].y); acc.w += bf16_hi(v[s].y);
  }
  *reinterpret_cast<uint2 *>(a.dq + (size_t(row) * a.H + h) * kHeadDim + lane * 4) =
      make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

template <int R>
cudaError_t launch_bwd_r(const CUtensorMap &tk, const CUtensorMap &tv, const BwdArgs &a,
                         int num_sms, cudaStream_t st) {
  auto kern = a.blk == 64 ? msa_backward_kernel<R, 64> : msa_backward_kernel<R, 128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem);
  if (e != cudaSuccess) return e;
  const int n_units = a.B * a.G * a.nb;
  const int grid = n_units < num_sms ? n_units : num_sms;
  kern<<<grid, kBwdThreads, kBwdSmem, st>>>(tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_delta(const BwdArgs &a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.L * a.H;
  if (rows == 0) return cudaSuccess;
  bwd_delta_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a.out, a.dout, a.delta, rows);
  return cudaGetLastError();
}

cudaError_t launch_backward(const CUtensorMap &tk, const CUtensorMap &tv, const BwdArgs &a,
                            int num_sms, cudaStream_t st) {
  const long long rows = (long long)a.Rc * a.H;
  if (rows == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(a.unit_ctr, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  switch (a.H / a.G) {
    case 1: e = launch_bwd_r<1>(tk, tv, a, num_sms, st); break;
    case 2: e = launch_bwd_r<2>(tk, tv, a, num_sms, st); break;
    case 4: e = launch_bwd_r<4>(tk, tv, a, num_sms, st); break;
    case 8: e = launch_bwd_r<8>(tk, tv, a, num_sms, st); break;
    case 16: e = launch_bwd_r<16>(tk, tv, a, num_sms, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (a.top_k <= 4)
    bwd_dq_reduce_kernel<4><<<grid, 256, 0, st>>>(a);
  else if (a.top_k <= 8)
    bwd_dq_reduce_kernel<8><<<grid, 256, 0, st>>>(a);
  else if (a.top_k <= 16)
    bwd_dq_reduce_kernel<16><<<grid, 256, 0, st>>>(a);
  else
    bwd_dq_reduce_kernel<32><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
