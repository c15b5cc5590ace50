// Decode step ("MiniMax M3 sparse attention" explainer, mlqm.cn/news/533796,
// §4.1: the new token scores the whole cache with the index branch and then
// attends only to its selected blocks, which cuts KV bandwidth by about an
// order of magnitude).  Everything here is bound by HBM bandwidth; the
// dominant stream is the k_idx cache scan (seq_len * d_idx * 2 bytes per
// sequence).
//
//   decode_index_kernel   one warp per (sequence, key block j < b_t):
//                         scores of the 128 keys against all G index
//                         queries with mma.sync m16n8k16 (N = 8 groups),
//                         then the per-group block max.  k_idx rows stream
//                         straight from HBM in 16-byte loads.
//   decode_topk_kernel    one CTA per (sequence, group): 16 warps scan
//                         segments of the block scores, one warp merges.
//   decode_attn_kernel    split over selected blocks: one CTA per
//                         (sequence, group, slot) computes the block's
//                         partial softmax for the R heads of the group.
//   decode_combine_kernel one warp per (sequence, head): merge <= top_k
//                         partials.
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

// A warp scores one 128-key block against the (up to 8) index queries of
// its sequence.  The MMA's k dimension is a fixed permutation of d_idx
// applied to both operands, chosen so that each lane reads whole 16-byte
// granules of k_idx: for k-step kk = 2m + h, lane (g4 = lane/4, c = lane%4)
// feeds d = 8(c + 4m) + 4h + {0,1} at k positions 2c, 2c+1 and
// d = 8(c + 4m) + 4h + {2,3} at k positions 2c+8, 2c+9.
template <int DI>
__global__ void __launch_bounds__(256) decode_index_kernel(const DecodeArgs a) {
  constexpr int NM = DI / 32;  // 16-byte granules per lane per key row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int j = blockIdx.x * 8 + warp;
  const int n = a.seq_lens[b];
  if (n < 1 || n > a.Lmax) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(a.status, 0, kStatusBadInput);
    return;
  }
  const int bt = (n - 1) / kBlock;
  if (bt + 1 <= a.top_k || j >= bt) return;
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
  const uint16_t *kbase = a.k_idx_cache + (size_t(b) * a.Lmax + size_t(j) * kBlock) * DI;
  float mx0 = -FLT_MAX, mx1 = -FLT_MAX;
#pragma unroll 2
  for (int rt = 0; rt < 8; ++rt) {
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
    mx0 = fmaxf(mx0, fmaxf(acc[0], acc[2]));
    mx1 = fmaxf(mx1, fmaxf(acc[1], acc[3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  if (lane < 4) {
    const int g0 = 2 * c, g1 = 2 * c + 1;
    if (g0 < a.G) a.scores[(size_t(b) * a.G + g0) * a.nb_max + j] = mx0;
    if (g1 < a.G) a.scores[(size_t(b) * a.G + g1) * a.nb_max + j] = mx1;
  }
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
  const int n = a.seq_lens[b];
  int32_t *out = a.sel + size_t(row) * a.top_k;
  if (n < 1 || n > a.Lmax) {
    if (warp == 0 && lane < a.top_k) out[lane] = -1;
    return;
  }
  const int bt = (n - 1) / kBlock;
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
      warp_topk_offer(m, cs, cj, lane < k1 && cj != INT_MAX && cs >= t0, k1);
    }
    warp_topk_write(m, bt, a.top_k, out);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// One CTA (128 threads) per (slot, group, sequence).  The block's K and V
// rows (128 x 256 B each, strided by G*d*2 bytes in the cache) are staged in
// shared memory with coalesced 16-byte cp.async, K and V as two groups so V
// streams in while the scores are computed.  Phase 1: thread = key, R dot
// products against the group's query heads.  Phase 2: thread = (d pair, key
// parity), sum_k p[h][k] v[k][d].
constexpr int kKPitch = kHeadDim + 8;  // bf16 elements per staged K row (272 B)

template <int R>
constexpr int decode_attn_smem() {
  return kBlock * kKPitch * 2 + kBlock * kHeadDim * 2 + kHeadDim * R * 4 + kBlock * R * 4 +
         R * kHeadDim * 4 + R * 4 * 4;
}

// q and p are kept head-minor ([d][R] and [key][R]) so one 16-byte shared
// load feeds four heads.
template <int R>
__device__ __forceinline__ void load_heads(const float *base, float (&v)[R]) {
  if constexpr (R % 4 == 0) {
#pragma unroll
    for (int h = 0; h < R; h += 4) {
      const float4 f = *reinterpret_cast<const float4 *>(base + h);
      v[h] = f.x; v[h + 1] = f.y; v[h + 2] = f.z; v[h + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int h = 0; h < R; ++h) v[h] = base[h];
  }
}

template <int R>
__global__ void __launch_bounds__(128) decode_attn_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  uint16_t *sK = reinterpret_cast<uint16_t *>(dsm);
  uint16_t *sV = sK + kBlock * kKPitch;
  float *s_q = reinterpret_cast<float *>(sV + kBlock * kHeadDim);   // [d][R]
  float *s_p = s_q + kHeadDim * R;                                   // [key][R]
  float(*s_acc)[kHeadDim] = reinterpret_cast<float(*)[kHeadDim]>(s_p + kBlock * R);
  float(*s_red)[4] = reinterpret_cast<float(*)[4]>(&s_acc[R][0]);
  const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int n = a.seq_lens[b];
  const int j = (n >= 1 && n <= a.Lmax) ? a.sel[(size_t(b) * a.G + g) * a.top_k + slot] : -1;
  const size_t prow0 = (size_t(b) * a.H + size_t(g) * R) * a.top_k + slot;
  if (j < 0) {
    if (tid < R) a.part_lse[prow0 + size_t(tid) * a.top_k] = -INFINITY;
    return;
  }
  const int t = n - 1;
  const int nvis = min(kBlock, t - j * kBlock + 1);
  const size_t row_stride = size_t(a.G) * kHeadDim;
  const uint16_t *kb = a.k_cache + ((size_t(b) * a.Lmax + size_t(j) * kBlock) * a.G + g) * kHeadDim;
  const uint16_t *vb = a.v_cache + ((size_t(b) * a.Lmax + size_t(j) * kBlock) * a.G + g) * kHeadDim;
  const uint32_t sK_u = static_cast<uint32_t>(__cvta_generic_to_shared(sK));
  const uint32_t sV_u = static_cast<uint32_t>(__cvta_generic_to_shared(sV));
#pragma unroll 4
  for (int it = 0; it < 16; ++it) {
    const int idx = it * 128 + tid, row = idx >> 4, gran = idx & 15;
    if (row < nvis) cp_async16(sK_u + (row * kKPitch + gran * 8) * 2, kb + row * row_stride + gran * 8);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll 4
  for (int it = 0; it < 16; ++it) {
    const int idx = it * 128 + tid, row = idx >> 4, gran = idx & 15;
    if (row < nvis) cp_async16(sV_u + (row * kHeadDim + gran * 8) * 2, vb + row * row_stride + gran * 8);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int x = tid; x < R * kHeadDim; x += 128) {
    const int h = x / kHeadDim, dd = x % kHeadDim;
    s_q[dd * R + h] = __bfloat162float(__ushort_as_bfloat16(a.q[(size_t(b) * a.H + g * R + h) * kHeadDim + dd]));
  }
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  // phase 1: scores (thread = key)
  const bool vis = tid < nvis;
  float sc[R];
#pragma unroll
  for (int h = 0; h < R; ++h) sc[h] = 0.f;
  if (vis) {
    const uint16_t *krow = sK + tid * kKPitch;
#pragma unroll 2
    for (int x = 0; x < 16; ++x) {
      const uint4 kv = *reinterpret_cast<const uint4 *>(krow + 8 * x);
      const float kf[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                           bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float qv[R];
        load_heads<R>(s_q + (8 * x + e) * R, qv);
#pragma unroll
        for (int h = 0; h < R; ++h) sc[h] = fmaf(qv[h], kf[e], sc[h]);
      }
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int h = 0; h < R; ++h) {
    float m = vis ? sc[h] : -FLT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[h][warp] = m;
  }
  __syncthreads();
  float mrow[R], lrow[R];
#pragma unroll
  for (int h = 0; h < R; ++h)
    mrow[h] = fmaxf(fmaxf(s_red[h][0], s_red[h][1]), fmaxf(s_red[h][2], s_red[h][3]));
  __syncthreads();
#pragma unroll
  for (int h = 0; h < R; ++h) {
    const float p = vis ? exp2f((sc[h] - mrow[h]) * a.scale_log2) : 0.f;
    s_p[tid * R + h] = p;
    float l = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) s_red[h][warp] = l;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
#pragma unroll
  for (int h = 0; h < R; ++h) lrow[h] = s_red[h][0] + s_red[h][1] + s_red[h][2] + s_red[h][3];
  // phase 2: O = P V over the visible keys
  const int dp = tid & 63, par = tid >> 6;
  float acc[R][2];
#pragma unroll
  for (int h = 0; h < R; ++h) acc[h][0] = acc[h][1] = 0.f;
#pragma unroll 4
  for (int k = par; k < nvis; k += 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(sV + k * kHeadDim + 2 * dp);
    const float v0 = bf16_lo(w), v1 = bf16_hi(w);
    float pv[R];
    load_heads<R>(s_p + k * R, pv);
#pragma unroll
    for (int h = 0; h < R; ++h) {
      acc[h][0] = fmaf(pv[h], v0, acc[h][0]);
      acc[h][1] = fmaf(pv[h], v1, acc[h][1]);
    }
  }
  if (par == 1) {
#pragma unroll
    for (int h = 0; h < R; ++h) { s_acc[h][2 * dp] = acc[h][0]; s_acc[h][2 * dp + 1] = acc[h][1]; }
  }
  __syncthreads();
  if (par == 0) {
#pragma unroll
    for (int h = 0; h < R; ++h) {
      const float inv = 1.f / lrow[h];
      float2 o2 = make_float2((acc[h][0] + s_acc[h][2 * dp]) * inv, (acc[h][1] + s_acc[h][2 * dp + 1]) * inv);
      *reinterpret_cast<float2 *>(a.part_o + (prow0 + size_t(h) * a.top_k) * kHeadDim + 2 * dp) = o2;
    }
  }
#pragma unroll
  for (int h = 0; h < R; ++h)
    if (tid == h) a.part_lse[prow0 + size_t(h) * a.top_k] = mrow[h] * a.scale + __logf(lrow[h]);
}

__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeArgs a) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);  // b*H + h
  const int lane = threadIdx.x & 31;
  if (row >= a.B * a.H) return;
  const size_t p0 = size_t(row) * a.top_k;
  const float my = lane < a.top_k ? a.part_lse[p0 + lane] : -INFINITY;
  float M = my;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (M > -INFINITY) {
    const float wm = (my > -INFINITY) ? __expf(my - M) : 0.f;
    wsum = wm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    for (int s = 0; s < a.top_k; ++s) {
      const float ws = __shfl_sync(0xffffffffu, wm, s);
      if (ws == 0.f) continue;
      const float4 v = *reinterpret_cast<const float4 *>(a.part_o + (p0 + s) * kHeadDim + lane * 4);
      acc[0] = fmaf(ws, v.x, acc[0]);
      acc[1] = fmaf(ws, v.y, acc[1]);
      acc[2] = fmaf(ws, v.z, acc[2]);
      acc[3] = fmaf(ws, v.w, acc[3]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint2 r;
  r.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  r.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  *reinterpret_cast<uint2 *>(a.out + size_t(row) * kHeadDim + lane * 4) = r;
}

template <int R>
cudaError_t launch_decode_attn(const DecodeArgs &a, cudaStream_t st) {
  constexpr int smem = decode_attn_smem<R>();
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<R>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<R><<<dim3(a.top_k, a.G, a.B), 128, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  const dim3 gi((a.nb_max + 7) / 8, a.B);
  if (a.d_idx == 64)
    decode_index_kernel<64><<<gi, 256, 0, st>>>(a);
  else
    decode_index_kernel<128><<<gi, 256, 0, st>>>(a);
  decode_topk_kernel<<<a.B * a.G, kTopkWarps * 32, 0, st>>>(a);
  cudaError_t e;
  switch (a.H / a.G) {
    case 1: e = launch_decode_attn<1>(a, st); break;
    case 2: e = launch_decode_attn<2>(a, st); break;
    case 4: e = launch_decode_attn<4>(a, st); break;
    case 8: e = launch_decode_attn<8>(a, st); break;
    case 16: e = launch_decode_attn<16>(a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<(a.B * a.H + 7) / 8, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
