// Main Branch, prefill: exact softmax attention over the selected blocks,
// organised key-block-outer ("MiniMax M3 sparse attention" explainer,
// mlqm.cn/news/533796, §2.2: gather the selected K/V blocks and run ordinary
// attention, all heads of a group sharing one selection; researchpapers.dev
// "MiniMax Sparse Attention", sections "机制" and "对工程团队的意义": query
// gathering and a reverse index; baguaai.com 稀疏注意力 MSA entry: "KV
// external aggregation Q").
//
// One work item = one (b, g, key block j) and up to 128/R queries that
// selected j, each with its R heads: a 128-row tile.  Per item:
//   TMA      K_j (128 x 128 bf16, 128B-swizzled) into the K/V buffer
//   gather   the tile's q rows (R heads of a query are 256*R contiguous
//            bytes) into a swizzled smem tile with cp.async
//   UMMA     S = Q K_j^T   (M=128, N=128, K=128) into TMEM
//   TMA      V_j into the K/V buffer, now that S has consumed K_j; the load
//            overlaps the softmax
//   softmax  thread r owns row r: mask s <= t, row max, exp2, row sum,
//            P = exp(...) as bf16 into smem (over the dead Q tile)
//   UMMA     O = P V_j into the same TMEM columns as S (V consumed MN-major
//            straight from its TMA tile)
//   store    O / l as a bf16 partial and lse = ln(sum exp(scale q.k)) per
//            (t, head, slot); a second kernel merges a row's <= top_k
//            partials.
// A CTA holds one 32 KB K/V buffer, one 32 KB Q/P tile and 128 TMEM columns,
// so three CTAs share an SM and their sequential phases overlap.  The next
// item's query list is fetched while this item computes, and its K and q
// rows are requested as soon as this item's second UMMA has consumed the
// shared tiles, so those loads overlap the partial-result stores.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kAttnCtasPerSm = 3;
constexpr int kSmemKV = 0;      // K tile, then V tile
constexpr int kSmemQ = 32768;   // Q tile, then P tile
constexpr int kSmemBar = 65536;
constexpr int kAttnSmem = kSmemBar + 64 + 1024 + 1024;  // bars, items, 2 lists, align slack

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

struct AttnItemWalk {  // thread 0's position in the CTA's item range
  int wb = 0, it_lo = 0, it_hi = 0, l_lo = 0, l_hi = 0;
};

// Gather the q rows of a work item into the swizzled Q tile: row = qi*R + hh,
// 16 granules of 16 B per row; rows past the item's queries are zeroed.
template <int R>
__device__ __forceinline__ void gather_q(const AttnArgs &a, uint32_t s_q, const int *list, int n,
                                         int b, int g, int tid) {
#pragma unroll 4
  for (int it = 0; it < 16; ++it) {
    const int idx = it * kAttnThreads + tid;
    const int row = idx >> 4;
    const int gran = idx & 15;
    const int qi = row / R;
    const int hh = row % R;
    const uint32_t dst = s_q + (gran >> 3) * 16384 + sw128_offset(row, gran & 7);
    if (qi < n) {
      const int t = list[qi] >> 5;
      const uint16_t *src =
          a.q + ((size_t(b) * a.L + t) * a.H + size_t(g) * R + hh) * kHeadDim + gran * 8;
      cp_async16(dst, src);
    } else {
      asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(dst), "r"(0) : "memory");
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kAttnThreads, kAttnCtasPerSm)
    msa_prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  constexpr int QPI = 128 / R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const uint32_t s_kv = smem_u32(smem + kSmemKV);
  const uint32_t s_q = smem_u32(smem + kSmemQ);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSmemBar);
  const uint32_t b_k = smem_u32(&bars[0]);
  const uint32_t b_v = smem_u32(&bars[1]);
  const uint32_t b_mma = smem_u32(&bars[2]);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(&bars[3]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  int *s_item = reinterpret_cast<int *>(smem + kSmemBar + 32);    // [2][4]: bgj, start, n, -
  int *s_list = reinterpret_cast<int *>(smem + kSmemBar + 64);    // [2][128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  if (tid == 0) {
    mbar_init(b_k, 1);
    mbar_init(b_v, 1);
    mbar_init(b_mma, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_holder;   // S, then O
  const uint32_t lane_off = uint32_t(warp * 32) << 16;

  const int n_bgj = a.B * a.G * a.nb;
  const int n_items = a.item_off[n_bgj];
  if (n_items > a.max_items && tid == 0) atomicCAS(a.status, 0, kStatusBadInput);
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
  uint32_t k_ph = 0, v_ph = 0, mma_ph = 0;

  // Each CTA takes a contiguous range of work items (ordered by (b, g, key
  // block), so consecutive items mostly read the same K/V block from L2).
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int w_begin = blockIdx.x * per;
  const int w_end = min(n_items, w_begin + per);
  AttnItemWalk wk;
  auto describe = [&](int w, int *dst) {  // thread 0: item w -> dst[0..2]
    while (w >= wk.it_hi) {
      ++wk.wb;
      wk.it_lo = wk.it_hi; wk.it_hi = a.item_off[wk.wb + 1];
      wk.l_lo = wk.l_hi; wk.l_hi = a.list_off[wk.wb + 1];
    }
    const int start = wk.l_lo + (w - wk.it_lo) * QPI;
    dst[0] = wk.wb;
    dst[1] = start;
    dst[2] = min(QPI, wk.l_hi - start);
  };
  // thread 0: one 128-key tile of K or V of block bgj into the K/V buffer
  auto issue_tile = [&](const CUtensorMap *tm, uint32_t bar, int bgj) {
    const int j = bgj % a.nb;
    const int bg = bgj / a.nb;
    const int g = bg % a.G;
    const int b = bg / a.G;
    mbar_arrive_expect_tx(bar, 32768);
    const int z = b * a.L + j * kBlock;
    tma_load_3d(s_kv, tm, bar, 0, g, z);
    tma_load_3d(s_kv + 16384, tm, bar, 64, g, z);
  };

  if (w_begin < w_end) {
    if (tid == 0) {
      int lo = 0, hi = n_bgj - 1;  // first bgj with item_off[bgj+1] > w_begin
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.item_off[mid] <= w_begin) lo = mid; else hi = mid - 1;
      }
      wk.wb = lo;
      wk.it_lo = a.item_off[lo]; wk.it_hi = a.item_off[lo + 1];
      wk.l_lo = a.list_off[lo]; wk.l_hi = a.list_off[lo + 1];
      describe(w_begin, s_item);
      issue_tile(&tm_k, b_k, s_item[0]);
    }
    __syncthreads();
    if (tid < s_item[2]) s_list[tid] = a.list[s_item[1] + tid];
    __syncthreads();
    gather_q<R>(a, s_q, s_list, s_item[2], s_item[0] / (a.nb * a.G), (s_item[0] / a.nb) % a.G, tid);
  }

  int buf = 0;
  for (int w = w_begin; w < w_end; ++w) {
    const int *it = s_item + 4 * buf;
    const int *lst = s_list + 128 * buf;
    const int bgj = it[0];
    const int n = it[2];
    const int j = bgj % a.nb;
    const int g = (bgj / a.nb) % a.G;
    const int b = bgj / (a.nb * a.G);
    const bool has_next = w + 1 < w_end;
    int *nit = s_item + 4 * (buf ^ 1);
    int *nlst = s_list + 128 * (buf ^ 1);
    if (has_next && tid == 0) describe(w + 1, nit);
    __syncthreads();
    // the next item's query list: loaded now, stored to shared memory after
    // this item's UMMAs, so its latency hides behind them
    const int n_next = has_next ? nit[2] : 0;
    const int next_entry = (tid < n_next) ? a.list[nit[1] + tid] : 0;

    // ---- this item's q rows have landed
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();

    // ---- S = Q K^T
    int ok_k = 1;
    if (tid == 0) {
      ok_k = mbar_wait(b_k, k_ph, abort_flag, a.status) ? 1 : 0;
      if (ok_k) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int c = kk >> 2;
          const uint32_t off = (kk & 3) * 32;
          umma_f16_ss(tmem_acc, sdesc_sw128(s_q + c * 16384 + off, 16, 1024),
                      sdesc_sw128(s_kv + c * 16384 + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(b_mma);
      }
    }
    k_ph ^= 1;
    // every exit decision below is taken by the whole CTA at one barrier
    if (__syncthreads_or(!ok_k)) break;
    const bool ok1 = mbar_wait(b_mma, mma_ph, abort_flag, a.status);
    mma_ph ^= 1;
    if (__syncthreads_or(!ok1)) break;
    tc_fence_after();
    // K has been consumed: bring V into the same buffer during the softmax
    if (tid == 0) issue_tile(&tm_v, b_v, bgj);

    // ---- softmax on row `tid`, two 64-column halves per pass
    const int qi = tid / R;
    const bool valid = qi < n;
    const int ent = valid ? lst[qi] : 0;
    const int t = ent >> 5;
    const int lim = valid ? (t - j * kBlock) : -1;  // last visible column
    float m = -FLT_MAX;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float t0[32], t1[32];
      tmem_ld32(tmem_acc + lane_off + h * 64, t0);
      tmem_ld32(tmem_acc + lane_off + h * 64 + 32, t1);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        if (h * 64 + x <= lim) m = fmaxf(m, t0[x]);
        if (h * 64 + 32 + x <= lim) m = fmaxf(m, t1[x]);
      }
    }
    const float mb = m * a.scale_log2;
    float l = 0.f;
    uint8_t *p_tile = smem + kSmemQ;
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      float sv[64];
      {
        float t0[32], t1[32];
        tmem_ld32(tmem_acc + lane_off + h * 64, t0);
        tmem_ld32(tmem_acc + lane_off + h * 64 + 32, t1);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) { sv[x] = t0[x]; sv[32 + x] = t1[x]; }
      }
#pragma unroll
      for (int gblk = 0; gblk < 8; ++gblk) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = gblk * 8 + e * 2;
          const int cg = h * 64 + c0;
          const float p0 = (cg <= lim) ? fast_exp2(fmaf(sv[c0], a.scale_log2, -mb)) : 0.f;
          const float p1 = (cg + 1 <= lim) ? fast_exp2(fmaf(sv[c0 + 1], a.scale_log2, -mb)) : 0.f;
          l += p0 + p1;
          w4[e] = pack_bf16x2(p0, p1);
        }
        *reinterpret_cast<uint4 *>(p_tile + h * 16384 + sw128_offset(tid, gblk)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O = P V (into the S columns: every thread has read S already)
    int ok_v = 1;
    if (tid == 0) {
      ok_v = mbar_wait(b_v, v_ph, abort_flag, a.status) ? 1 : 0;
      if (ok_v) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int c = kk >> 2;
          const uint32_t off = (kk & 3) * 32;
          umma_f16_ss(tmem_acc, sdesc_sw128(s_q + c * 16384 + off, 16, 1024),
                      sdesc_sw128(s_kv + kk * 2048, 16384, 1024), idesc_o, kk > 0);
        }
        umma_commit(b_mma);
      }
    }
    v_ph ^= 1;
    if (__syncthreads_or(!ok_v)) break;
    const bool ok2 = mbar_wait(b_mma, mma_ph, abort_flag, a.status);
    mma_ph ^= 1;
    if (__syncthreads_or(!ok2)) break;
    tc_fence_after();

    // ---- the shared tiles are free: request the next item's K and q rows
    if (tid < n_next) nlst[tid] = next_entry;
    __syncthreads();
    if (has_next) {
      if (tid == 0) issue_tile(&tm_k, b_k, nit[0]);
      gather_q<R>(a, s_q, nlst, nit[2], nit[0] / (a.nb * a.G), (nit[0] / a.nb) % a.G, tid);
    }

    // ---- store the normalised partial and its lse.  tcgen05.ld is a
    // warp-wide (.sync.aligned) instruction: every thread loads, only rows
    // holding a query store.
    {
      const int slot = ent & 31;
      const int hh = tid % R;
      const bool store = valid && lim >= 0;
      const float inv = store ? 1.f / l : 0.f;
      const size_t prow =
          ((size_t(b) * a.Lc + (t - a.t0)) * a.H + size_t(g) * R + hh) * a.top_k + slot;
      uint4 *dst = reinterpret_cast<uint4 *>(a.part_o + prow * kHeadDim);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float o0[32], o1[32];
        tmem_ld32(tmem_acc + lane_off + h * 64, o0);
        tmem_ld32(tmem_acc + lane_off + h * 64 + 32, o1);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[h * 8 + x] = make_uint4(pack_bf16x2(o0[8 * x] * inv, o0[8 * x + 1] * inv),
                                        pack_bf16x2(o0[8 * x + 2] * inv, o0[8 * x + 3] * inv),
                                        pack_bf16x2(o0[8 * x + 4] * inv, o0[8 * x + 5] * inv),
                                        pack_bf16x2(o0[8 * x + 6] * inv, o0[8 * x + 7] * inv));
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[h * 8 + 4 + x] = make_uint4(pack_bf16x2(o1[8 * x] * inv, o1[8 * x + 1] * inv),
                                            pack_bf16x2(o1[8 * x + 2] * inv, o1[8 * x + 3] * inv),
                                            pack_bf16x2(o1[8 * x + 4] * inv, o1[8 * x + 5] * inv),
                                            pack_bf16x2(o1[8 * x + 6] * inv, o1[8 * x + 7] * inv));
        }
      }
      if (valid) a.part_lse[prow] = store ? m * a.scale + __logf(l) : -INFINITY;
    }
    tc_fence_before();
    __syncthreads();
    buf ^= 1;
  }

  cp_async_wait_all();   // nothing may still be landing in shared memory
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, 128);
  }
}

template <int R>
cudaError_t launch_attn_r(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                          int num_sms, cudaStream_t st) {
  auto kern = msa_prefill_attn_kernel<R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  int grid = kAttnCtasPerSm * num_sms;
  if (a.max_items < grid) grid = a.max_items > 0 ? a.max_items : 1;
  kern<<<grid, kAttnThreads, kAttnSmem, st>>>(tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attn(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                                int num_sms, cudaStream_t st) {
  const int R = a.H / a.G;
  switch (R) {
    case 1: return launch_attn_r<1>(tk, tv, a, num_sms, st);
    case 2: return launch_attn_r<2>(tk, tv, a, num_sms, st);
    case 4: return launch_attn_r<4>(tk, tv, a, num_sms, st);
    case 8: return launch_attn_r<8>(tk, tv, a, num_sms, st);
    case 16: return launch_attn_r<16>(tk, tv, a, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- combine
namespace {

// One warp per (b, t, h): merge the row's partials (normalised o_s, lse_s)
// into o = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M), M = max lse_s.
// All of a lane's partial-row loads (4 of the d values of each slot) and its
// lse load are issued before any reduction, so a row costs one memory round
// trip after its selection row is known.
template <int KCAP>
__global__ void __launch_bounds__(256) msa_combine_kernel(const CombineArgs a) {
  const long long wrow = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)a.B * a.Lc * a.H;
  if (wrow >= n_rows) return;
  const int h = (int)(wrow % a.H);
  const long long bt = wrow / a.H;
  const int tl = (int)(bt % a.Lc);
  const int b = (int)(bt / a.Lc);
  const int t = a.t0 + tl;
  const int g = h / (a.H / a.G);
  const int32_t *sel = a.sel + ((size_t(b) * a.G + g) * a.L + t) * a.top_k;
  const size_t prow0 = (((size_t)b * a.Lc + tl) * a.H + h) * a.top_k;
  const bool mine = lane < a.top_k && sel[lane] >= 0;
  const unsigned vmask = __ballot_sync(0xffffffffu, mine);
  uint2 v[KCAP];
#pragma unroll
  for (int s = 0; s < KCAP; ++s) {
    v[s] = make_uint2(0u, 0u);
    if ((vmask >> s) & 1u)
      v[s] = __ldcs(reinterpret_cast<const uint2 *>(a.part_o + (prow0 + s) * kHeadDim + lane * 4));
  }
  const float my_lse = mine ? __ldcs(a.part_lse + prow0 + lane) : -INFINITY;
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
  uint2 r;
  r.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  r.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  *reinterpret_cast<uint2 *>(a.out + (((size_t)b * a.L + t) * a.H + h) * kHeadDim + lane * 4) = r;
  if (a.lse && lane == 0) a.lse[((size_t)b * a.L + t) * a.H + h] = (wsum > 0.f) ? M + __logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
  const long long n_rows = (long long)a.B * a.Lc * a.H;
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
