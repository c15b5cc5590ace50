// C ABI of the MSA library (see include/msa.h): argument checks, workspace
// planning, TMA descriptor encoding and kernel dispatch.  No allocation, no
// synchronisation except in msa_read_status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/msa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char *where) {
  return fail(MSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- shape checks ---------------------------------------------------------
int check_params(const msa_params *p, bool decode) {
  if (!p) return fail(MSA_ERR_INVALID_ARG, "params is NULL");
  if (p->B < 0 || p->L < 0 || p->H <= 0 || p->G <= 0 || p->d <= 0 || p->d_idx <= 0 ||
      p->block <= 0 || p->top_k <= 0)
    return fail(MSA_ERR_INVALID_ARG, "negative or zero size in params");
  if (!std::isfinite(p->scale) || p->scale < 0.f)
    return fail(MSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (p->d != 128) return fail(MSA_ERR_UNSUPPORTED, "d=%d (supported: 128)", p->d);
  if (p->d_idx != 64 && p->d_idx != 128)
    return fail(MSA_ERR_UNSUPPORTED, "d_idx=%d (supported: 64, 128)", p->d_idx);
  if (p->block != 128) return fail(MSA_ERR_UNSUPPORTED, "block=%d (supported: 128)", p->block);
  if (p->top_k > msa::kMaxTopK)
    return fail(MSA_ERR_UNSUPPORTED, "top_k=%d (supported: 1..32)", p->top_k);
  if (p->H % p->G != 0) return fail(MSA_ERR_INVALID_ARG, "H=%d not a multiple of G=%d", p->H, p->G);
  const int r = p->H / p->G;
  if (r != 1 && r != 2 && r != 4 && r != 8 && r != 16)
    return fail(MSA_ERR_UNSUPPORTED, "H/G=%d (supported: 1,2,4,8,16)", r);
  if (p->L % 128 != 0) return fail(MSA_ERR_UNSUPPORTED, "L=%d not a multiple of 128", p->L);
  if (decode && p->G > 8) return fail(MSA_ERR_UNSUPPORTED, "decode supports G <= 8 (G=%d)", p->G);
  if ((long long)p->B * p->L > (1LL << 26))
    return fail(MSA_ERR_UNSUPPORTED, "B*L=%lld above 2^26", (long long)p->B * p->L);
  if (p->chunk < 0 || p->chunk % 128 != 0)
    return fail(MSA_ERR_INVALID_ARG, "chunk=%d must be 0 or a positive multiple of 128", p->chunk);
  return MSA_OK;
}

float eff_scale(const msa_params *p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(float(p->d));
}

// ---- workspace plans --------------------------------------------------------
// Prefill attention processes queries in chunks of Lc so that the partial
// results (bf16, one 128-wide row per selected (query, head, slot)) stay
// within a fixed budget.  Every chunk reads the K/V blocks its queries
// select, which for long inputs is most of K/V, so fewer, larger chunks
// cut K/V re-reads: 16 GiB of partials is 9 chunks at 1M tokens, H=32,
// top_k=16 (a small share of HBM on this part).
constexpr size_t kPartialBudget = size_t(16) << 30;  // 16 GiB

int prefill_chunk(const msa_params *p) {
  const size_t per_q = size_t(p->B) * p->H * p->top_k * (p->d * 2 + 4);
  long long lc = per_q ? (long long)(kPartialBudget / per_q) : p->L;
  lc = (lc / 128) * 128;
  if (lc < 128) lc = 128;
  if (p->chunk > 0 && p->chunk < lc) lc = p->chunk;
  if (lc > p->L) lc = p->L;
  return (int)lc;
}

struct AttnWs {
  size_t cnt, list_off, item_off, list, pos_of, part_o, part_lse, end;
  int Lc;
};
AttnWs attn_ws(const msa_params *p, size_t base) {
  AttnWs w;
  w.Lc = prefill_chunk(p);
  const size_t nb = size_t(p->L) / 128;
  const size_t nbgj = size_t(p->B) * p->G * nb;
  size_t o = base;
  w.cnt = o; o = align_up(o + 4 * nbgj);
  w.list_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.item_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.list = o; o = align_up(o + 4 * size_t(p->B) * p->G * w.Lc * p->top_k);
  w.pos_of = o; o = align_up(o + 4 * size_t(p->B) * p->G * w.Lc * p->top_k);
  w.part_o = o; o = align_up(o + 2 * size_t(p->B) * w.Lc * p->H * p->top_k * p->d);
  w.part_lse = o; o = align_up(o + 4 * size_t(p->B) * w.Lc * p->H * p->top_k);
  w.end = o;
  return w;
}

// Backward: D = do . o per row; per query chunk (the prefill's chunk length)
// a reverse index and one bf16 dq partial row per (query, head, slot); with
// more than one chunk, fp32 dk/dv accumulators over the whole sequence.
struct BwdWs {
  size_t cnt, list_off, item_off, list, pos_of, delta, part_dq, acc_dk, acc_dv, end;
  int Lc;
};
BwdWs bwd_ws(const msa_params *p) {
  BwdWs w;
  w.Lc = prefill_chunk(p);
  const size_t nb = size_t(p->L) / 128;
  const size_t nbgj = size_t(p->B) * p->G * nb;
  const size_t entries = size_t(p->B) * p->G * w.Lc * p->top_k;
  size_t o = msa::kWsHeader;
  w.cnt = o; o = align_up(o + 4 * nbgj);
  w.list_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.item_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.list = o; o = align_up(o + 4 * entries);
  w.pos_of = o; o = align_up(o + 4 * entries);
  w.delta = o; o = align_up(o + 4 * size_t(p->B) * p->L * p->H);
  w.part_dq = o; o = align_up(o + 2 * entries * (p->H / p->G) * size_t(p->d));
  w.acc_dk = w.acc_dv = 0;
  if (w.Lc < p->L) {
    const size_t kv = 4 * size_t(p->B) * p->L * p->G * p->d;
    w.acc_dk = o; o = align_up(o + kv);
    w.acc_dv = o; o = align_up(o + kv);
  }
  w.end = o;
  return w;
}

struct DecWs {
  size_t scores, sel, part_o, part_lse, end;
};
DecWs dec_ws(const msa_params *p) {
  DecWs w;
  const size_t nb = size_t(p->L) / 128;
  size_t o = msa::kWsHeader;
  w.scores = o; o = align_up(o + 4 * size_t(p->B) * p->G * nb);
  w.sel = o; o = align_up(o + 4 * size_t(p->B) * p->G * p->top_k);
  w.part_o = o; o = align_up(o + 4 * size_t(p->B) * p->H * p->top_k * p->d);
  w.part_lse = o; o = align_up(o + 4 * size_t(p->B) * p->H * p->top_k);
  w.end = o;
  return w;
}

size_t forward_sel_bytes(const msa_params *p) {
  return align_up(4 * size_t(p->B) * p->G * p->L * p->top_k);
}

int check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(MSA_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign)
    return fail(MSA_ERR_WORKSPACE, "workspace not %zu-byte aligned", kAlign);
  if (ws_bytes < need)
    return fail(MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
  return MSA_OK;
}

// ---- TMA descriptors --------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 tensor of `rank` dims (innermost first), 128B swizzle, box as given.
int make_tmap(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
              const uint64_t *strides_bytes, const uint32_t *box) {
  auto fn = encode_fn();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  uint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
                  strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MSA_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int *status_ptr(void *ws) { return reinterpret_cast<int *>(ws); }

// ---- the operations --------------------------------------------------------
// Query-side geometry: q, q_idx, sel and out hold Lq rows per sequence, row
// 0 being position tq0 (Lq = L, tq0 = 0 for a whole sequence); k, v and
// k_idx hold p->L rows per sequence.
struct QGeom {
  int Lq, tq0;
};
QGeom whole(const msa_params *p) { return QGeom{p->L, 0}; }

// Index branch for the query tiles of tokens [t_lo, t_hi) (multiples of 128
// within [tq0, tq0 + Lq)).
int run_index_select(const msa_params *p, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                     int32_t *sel, float *block_scores, void *ws, cudaStream_t st, QGeom qg,
                     int t_lo, int t_hi) {
  const int nb = p->L / 128;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[3] = {uint64_t(p->d_idx), uint64_t(p->G), uint64_t(p->B) * qg.Lq};
    const uint64_t str[2] = {uint64_t(p->d_idx) * 2, uint64_t(p->d_idx) * 2 * p->G};
    const uint32_t box[3] = {64, 1, 128};
    int rc = make_tmap(&tq, q_idx, 3, dims, str, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {uint64_t(p->d_idx), uint64_t(p->B) * p->L};
    const uint64_t str[1] = {uint64_t(p->d_idx) * 2};
    const uint32_t box[2] = {64, 128};
    int rc = make_tmap(&tk, k_idx, 2, dims, str, box);
    if (rc) return rc;
  }
  msa::IndexArgs a;
  a.B = p->B; a.L = p->L; a.G = p->G; a.nb = nb; a.top_k = p->top_k; a.d_idx = p->d_idx;
  a.Lq = qg.Lq; a.tq0 = qg.tq0;
  a.write_scores = block_scores ? 1 : 0;
  a.i_hi = t_hi / 128;
  a.n_items = p->B * (t_hi / 128 - t_lo / 128) * (p->G / msa::index_groups_per_cta(p->G, p->top_k));
  a.sel = sel;
  a.scores = block_scores;
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_index_kernel(tq, tk, a, num_sms(), st);
  if (e != cudaSuccess) return cuda_fail(e, "index kernel launch");
  if (block_scores) {
    msa::TopkArgs t;
    t.B = p->B; t.G = p->G; t.L = p->L; t.nb = nb; t.top_k = p->top_k;
    t.scores = block_scores;
    t.sel = sel;
    e = msa::launch_topk_kernel(t, st);
    if (e != cudaSuccess) return cuda_fail(e, "top-k kernel launch");
  }
  return MSA_OK;
}

// Where a finished query chunk's output rows go next (msa_forward_host):
// after the chunk's merge, `copy` waits for it and downloads the rows.
struct ChunkSink {
  cudaStream_t copy;
  cudaEvent_t ev;
  msa_bf16 *out_h;
  float *lse_h;
};

// Tensor maps and workspace layout shared by the query chunks of one call.
struct AttnPlan {
  CUtensorMap tk, tv;
  AttnWs w;
  int nb, qpi, sms;
  float scale;
  QGeom qg;
};

int plan_attn(const msa_params *p, const msa_bf16 *k, const msa_bf16 *v, size_t ws_base,
              QGeom qg, AttnPlan *pl) {
  pl->nb = p->L / 128;
  pl->qg = qg;
  pl->w = attn_ws(p, ws_base);
  const uint64_t dims[3] = {uint64_t(p->d), uint64_t(p->G), uint64_t(p->B) * p->L};
  const uint64_t str[2] = {uint64_t(p->d) * 2, uint64_t(p->d) * 2 * p->G};
  const uint32_t box[3] = {64, 1, 128};
  int rc = make_tmap(&pl->tk, k, 3, dims, str, box);
  if (rc) return rc;
  rc = make_tmap(&pl->tv, v, 3, dims, str, box);
  if (rc) return rc;
  pl->qpi = 128 / (p->H / p->G);
  pl->scale = eff_scale(p);
  pl->sms = num_sms();
  return MSA_OK;
}

// One query chunk [t0, t0 + Lc): reverse index, attention, merge; then,
// with a sink, the download of the chunk's output rows.
int run_attn_chunk(const msa_params *p, const AttnPlan &pl, const msa_bf16 *q, const int32_t *sel,
                   msa_bf16 *out, float *lse, void *ws, int t0, int Lc, cudaStream_t st,
                   const ChunkSink *sink) {
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  const AttnWs &w = pl.w;
  msa::RevIdxArgs ra;
  ra.B = p->B; ra.G = p->G; ra.L = p->L; ra.nb = pl.nb; ra.top_k = p->top_k; ra.qpi = pl.qpi;
  ra.Lq = pl.qg.Lq; ra.tq0 = pl.qg.tq0;
  ra.t0 = t0; ra.Lc = Lc;
  ra.sel = sel;
  ra.cnt = reinterpret_cast<int32_t *>(wsb + w.cnt);
  ra.list_off = reinterpret_cast<int32_t *>(wsb + w.list_off);
  ra.item_off = reinterpret_cast<int32_t *>(wsb + w.item_off);
  ra.list = reinterpret_cast<int32_t *>(wsb + w.list);
  ra.pos_of = reinterpret_cast<int32_t *>(wsb + w.pos_of);
  ra.status = status_ptr(ws);
  cudaError_t e = msa::launch_revidx(ra, st);
  if (e != cudaSuccess) return cuda_fail(e, "reverse index launch");
  msa::AttnArgs aa;
  aa.B = p->B; aa.L = p->L; aa.H = p->H; aa.G = p->G; aa.nb = pl.nb; aa.top_k = p->top_k;
  aa.Lq = pl.qg.Lq; aa.tq0 = pl.qg.tq0;
  aa.scale = pl.scale;
  aa.scale_log2 = pl.scale * 1.4426950408889634f;
  aa.t0 = t0; aa.Lc = Lc;
  const long long max_items =
      (long long)p->B * p->G * Lc * p->top_k / pl.qpi + (long long)p->B * p->G * pl.nb;
  aa.max_items = (int)max_items;
  aa.q = q;
  aa.list = ra.list; aa.list_off = ra.list_off; aa.item_off = ra.item_off;
  aa.part_o = reinterpret_cast<uint16_t *>(wsb + w.part_o);
  aa.part_lse = reinterpret_cast<float *>(wsb + w.part_lse);
  aa.status = status_ptr(ws);
  e = msa::launch_prefill_attn(pl.tk, pl.tv, aa, pl.sms, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
  msa::CombineArgs ca;
  ca.B = p->B; ca.L = p->L; ca.H = p->H; ca.G = p->G; ca.top_k = p->top_k;
  ca.Lq = pl.qg.Lq; ca.tq0 = pl.qg.tq0;
  ca.t0 = t0; ca.Lc = Lc;
  ca.sel = sel;
  ca.pos_of = ra.pos_of;
  ca.part_o = aa.part_o; ca.part_lse = aa.part_lse;
  ca.out = out; ca.lse = lse;
  e = msa::launch_combine(ca, st);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  if (sink) {
    e = cudaEventRecord(sink->ev, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sink->copy, sink->ev, 0);
    if (e != cudaSuccess) return cuda_fail(e, "chunk event");
    const size_t row = size_t(p->H) * p->d;   // elements of one token's output
    for (int b = 0; b < p->B && e == cudaSuccess; ++b) {
      const size_t qr = size_t(b) * pl.qg.Lq + (t0 - pl.qg.tq0);   // query-side row of t0
      const size_t off = qr * row;
      e = cudaMemcpyAsync(sink->out_h + off, out + off, size_t(Lc) * row * 2,
                          cudaMemcpyDeviceToHost, sink->copy);
      if (e == cudaSuccess && sink->lse_h) {
        const size_t lo = qr * p->H;
        e = cudaMemcpyAsync(sink->lse_h + lo, lse + lo, size_t(Lc) * p->H * 4,
                            cudaMemcpyDeviceToHost, sink->copy);
      }
    }
    if (e != cudaSuccess) return cuda_fail(e, "output download");
  }
  return MSA_OK;
}

// Main branch for the queries of positions [qg.tq0, qg.tq0 + qg.Lq).
int run_prefill_attn(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k,
                     const msa_bf16 *v, const int32_t *sel, msa_bf16 *out, float *lse, void *ws,
                     size_t ws_base, cudaStream_t st, QGeom qg) {
  AttnPlan pl;
  int rc = plan_attn(p, k, v, ws_base, qg, &pl);
  if (rc) return rc;
  const int t_end = qg.tq0 + qg.Lq;
  for (int t0 = qg.tq0; t0 < t_end; t0 += pl.w.Lc) {
    const int Lc = (t_end - t0) < pl.w.Lc ? (t_end - t0) : pl.w.Lc;
    rc = run_attn_chunk(p, pl, q, sel, out, lse, ws, t0, Lc, st, nullptr);
    if (rc) return rc;
  }
  return MSA_OK;
}

// Events and download stream of msa_forward_host, created once per device.
// Each record is followed at once by the wait that consumes it, under the
// mutex, so reusing one event per role is safe.
struct HostEvents {
  cudaEvent_t idx_in = nullptr, all_in = nullptr, chunk = nullptr, done = nullptr;
  cudaStream_t down = nullptr;   // output downloads (the other PCIe direction)
  unsigned long long ctx_id = 0; // context they were created in
};
constexpr int kMaxDevices = 64;
std::mutex g_host_mu;
HostEvents g_host_ev[kMaxDevices];

int host_events(HostEvents **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device %d", dev);
  HostEvents &h = g_host_ev[dev];
  // Events and streams belong to the context they were created in; after the
  // device's context is rebuilt (cudaDeviceReset) they are created anew.
  unsigned long long id = 0;
  e = cudaSetDevice(dev);   // makes the device's primary context current (creating it if needed)
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  if (msa::current_context_id(&id) && id != h.ctx_id) {
    h = HostEvents{};
    h.ctx_id = id;
  }
  cudaEvent_t *evs[4] = {&h.idx_in, &h.all_in, &h.chunk, &h.done};
  for (cudaEvent_t *ev : evs) {
    if (*ev) continue;
    e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreateWithFlags");
  }
  if (!h.down) {
    e = cudaStreamCreateWithFlags(&h.down, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
  }
  *out = &h;
  return MSA_OK;
}

// FP8 caches of a decode step: E4M3 codes with their scales (null: bf16).
struct Fp8Caches {
  const uint8_t *k_idx8 = nullptr;
  const float *k_idx_scale = nullptr;
  const uint8_t *k8 = nullptr, *v8 = nullptr;
  const float *k_scale = nullptr, *v_scale = nullptr;
};

// Decode step.  The index-key cache is bf16 (k_idx_cache) or FP8
// (f8.k_idx8 + scale); K/V are bf16 (k_cache, v_cache) or FP8 (f8.k8/v8 +
// scales).
int run_decode(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
               const msa_bf16 *k_cache, const msa_bf16 *v_cache, const msa_bf16 *k_idx_cache,
               const Fp8Caches &f8, const int32_t *seq_lens, msa_bf16 *out, int32_t *sel,
               void *ws, size_t ws_bytes, cudaStream_t st) {
  const uint8_t *k_idx8 = f8.k_idx8;
  const float *k_idx_scale = f8.k_idx_scale;
  int rc = check_params(p, true);
  if (rc) return rc;
  if (p->B == 0) return MSA_OK;
  if (p->L == 0) return fail(MSA_ERR_INVALID_ARG, "decode needs a cache (L = Lmax > 0)");
  const bool kv8 = f8.k8 != nullptr;
  if (!q || !q_idx || !seq_lens || !out || (!k_idx_cache && !k_idx8) || (k_idx8 && !k_idx_scale) ||
      (!kv8 && (!k_cache || !v_cache)) ||
      (kv8 && (!f8.v8 || !f8.k_scale || !f8.v_scale)))
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  auto al4 = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
  if (kv8 && (!aligned16(f8.k8) || !aligned16(f8.v8) || !al4(f8.k_scale) || !al4(f8.v_scale)))
    return fail(MSA_ERR_INVALID_ARG, "FP8 caches must be 16-byte aligned (scales 4-byte)");
  if (!aligned16(q) || !aligned16(q_idx) || (k_cache && !aligned16(k_cache)) ||
      (v_cache && !aligned16(v_cache)) ||
      (k_idx_cache && !aligned16(k_idx_cache)) || (k_idx8 && !aligned16(k_idx8)) ||
      (k_idx_scale && (reinterpret_cast<uintptr_t>(k_idx_scale) & 3u)) || !aligned16(out) ||
      (sel && !aligned16(sel)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (scales 4-byte)");
  const DecWs w = dec_ws(p);
  rc = check_ws(ws, ws_bytes, w.end);
  if (rc) return rc;
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  msa::DecodeArgs a;
  a.B = p->B; a.Lmax = p->L; a.H = p->H; a.G = p->G; a.d_idx = p->d_idx;
  a.nb_max = p->L / 128; a.top_k = p->top_k;
  a.scale = eff_scale(p);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.q = q; a.q_idx = q_idx; a.k_cache = k_cache; a.v_cache = v_cache; a.k_idx_cache = k_idx_cache;
  a.k_idx8 = k_idx8; a.k_idx_scale = k_idx_scale;
  a.k8 = f8.k8; a.v8 = f8.v8; a.k_scale = f8.k_scale; a.v_scale = f8.v_scale;
  a.seq_lens = seq_lens;
  a.scores = reinterpret_cast<float *>(wsb + w.scores);
  a.sel = sel ? sel : reinterpret_cast<int32_t *>(wsb + w.sel);
  a.part_o = reinterpret_cast<float *>(wsb + w.part_o);
  a.part_lse = reinterpret_cast<float *>(wsb + w.part_lse);
  a.out = out;
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_decode(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return MSA_OK;
}

}  // namespace

namespace msa {
// Records an error message for msa_last_error() from other translation units.
int report_error(int code, const char *msg) { return fail(code, "%s", msg); }

bool current_context_id(unsigned long long *id) {
  // Driver entry points resolved through the runtime, so the library needs
  // no link against libcuda.
  using CtxGetCurrentFn = CUresult (*)(CUcontext *);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}
}  // namespace msa

extern "C" {

const char *msa_last_error(void) { return g_err; }

const char *msa_version(void) { return "msa-b200 0.1 (sm_100a)"; }

size_t msa_workspace_bytes(const msa_params *p, int op) {
  g_err[0] = 0;
  if (check_params(p, op == MSA_OP_DECODE) != MSA_OK) return 0;
  switch (op) {
    case MSA_OP_INDEX_SELECT: return msa::kWsHeader;
    case MSA_OP_PREFILL_ATTN: return attn_ws(p, msa::kWsHeader).end;
    case MSA_OP_DECODE: return dec_ws(p).end;
    case MSA_OP_FORWARD: return attn_ws(p, msa::kWsHeader + forward_sel_bytes(p)).end;
    case MSA_OP_BACKWARD: return bwd_ws(p).end;
    default: fail(MSA_ERR_INVALID_ARG, "unknown op %d", op); return 0;
  }
}

int msa_prefill_chunk_len(const msa_params *p) {
  g_err[0] = 0;
  if (check_params(p, false) != MSA_OK) return 0;
  return p->L > 0 ? prefill_chunk(p) : 0;
}

int msa_read_status(void *ws, msa_stream stream) {
  g_err[0] = 0;
  if (!ws) return fail(MSA_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading device status");
  if (v != 0) {
    e = cudaMemsetAsync(ws, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    return fail(v, "device reported status %d (%s)", v,
                v == MSA_ERR_DEVICE_TIMEOUT ? "a bounded wait ran out" : "invalid device input");
  }
  return MSA_OK;
}

int msa_index_select(const msa_params *p, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                     int32_t *sel, float *block_scores, void *ws, size_t ws_bytes,
                     msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q_idx || !k_idx || !sel) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(sel) ||
      (block_scores && !aligned16(block_scores)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  rc = check_ws(ws, ws_bytes, msa::kWsHeader);
  if (rc) return rc;
  return run_index_select(p, q_idx, k_idx, sel, block_scores, ws,
                          reinterpret_cast<cudaStream_t>(stream), whole(p), 0, p->L);
}

int msa_sparse_attn_prefill(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k,
                            const msa_bf16 *v, const int32_t *sel, msa_bf16 *out, float *lse,
                            void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k || !v || !sel || !out) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(sel) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t need = attn_ws(p, msa::kWsHeader).end;
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  return run_prefill_attn(p, q, k, v, sel, out, lse, ws, msa::kWsHeader,
                          reinterpret_cast<cudaStream_t>(stream), whole(p));
}

int msa_forward(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k, const msa_bf16 *v,
                const msa_bf16 *q_idx, const msa_bf16 *k_idx, msa_bf16 *out, int32_t *sel,
                float *lse, void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k || !v || !q_idx || !k_idx || !out)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) ||
      !aligned16(k_idx) || !aligned16(out) || (sel && !aligned16(sel)) || (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t base = msa::kWsHeader + forward_sel_bytes(p);
  rc = check_ws(ws, ws_bytes, attn_ws(p, base).end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t *s = sel ? sel : reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + msa::kWsHeader);
  rc = run_index_select(p, q_idx, k_idx, s, nullptr, ws, st, whole(p), 0, p->L);
  if (rc) return rc;
  return run_prefill_attn(p, q, k, v, s, out, lse, ws, base, st, whole(p));
}

int msa_forward_cached(const msa_params *p, int t0, int n, const msa_bf16 *q,
                       const msa_bf16 *q_idx, const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                       const msa_bf16 *k_idx_cache, msa_bf16 *out, int32_t *sel, float *lse,
                       void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (t0 < 0 || n < 0 || t0 % 128 != 0 || n % 128 != 0 || (long long)t0 + n > p->L)
    return fail(MSA_ERR_INVALID_ARG, "t0=%d n=%d: need multiples of 128 with t0 + n <= L=%d", t0,
                n, p->L);
  if (p->B == 0 || n == 0) return MSA_OK;
  if (!q || !q_idx || !k_cache || !v_cache || !k_idx_cache || !out)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(q_idx) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(k_idx_cache) || !aligned16(out) || (sel && !aligned16(sel)) ||
      (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t base = msa::kWsHeader + forward_sel_bytes(p);
  rc = check_ws(ws, ws_bytes, attn_ws(p, base).end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const QGeom qg{n, t0};
  int32_t *s = sel ? sel : reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + msa::kWsHeader);
  rc = run_index_select(p, q_idx, k_idx_cache, s, nullptr, ws, st, qg, t0, t0 + n);
  if (rc) return rc;
  return run_prefill_attn(p, q, k_cache, v_cache, s, out, lse, ws, base, st, qg);
}

int msa_forward_cached_varlen(const msa_params *p, const int32_t *t0, const int32_t *n,
                              const msa_bf16 *q, const msa_bf16 *q_idx, const msa_bf16 *k_cache,
                              const msa_bf16 *v_cache, const msa_bf16 *k_idx_cache,
                              msa_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                              msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0) return MSA_OK;
  if (!t0 || !n) return fail(MSA_ERR_INVALID_ARG, "NULL t0 or n (host arrays)");
  for (int b = 0; b < p->B; ++b)
    if (t0[b] < 0 || n[b] < 0 || t0[b] % 128 || n[b] % 128 || (long long)t0[b] + n[b] > p->L)
      return fail(MSA_ERR_INVALID_ARG, "sequence %d: t0=%d n=%d (multiples of 128, t0+n <= L=%d)",
                  b, t0[b], n[b], p->L);
  msa_params p1 = *p;
  p1.B = 1;
  const size_t kv_rows = size_t(p->L);   // cache rows per sequence
  long long row0 = 0;
  for (int b = 0; b < p->B; ++b) {
    if (n[b] > 0) {
      rc = msa_forward_cached(&p1, t0[b], n[b], q + size_t(row0) * p->H * p->d,
                              q_idx + size_t(row0) * p->G * p->d_idx,
                              k_cache + size_t(b) * kv_rows * p->G * p->d,
                              v_cache + size_t(b) * kv_rows * p->G * p->d,
                              k_idx_cache + size_t(b) * kv_rows * p->d_idx,
                              out + size_t(row0) * p->H * p->d, nullptr,
                              lse ? lse + size_t(row0) * p->H : nullptr, ws, ws_bytes, stream);
      if (rc) return rc;
    }
    row0 += n[b];
  }
  return MSA_OK;
}

int msa_forward_host(const msa_params *p, const msa_bf16 *q_h, const msa_bf16 *k_h,
                     const msa_bf16 *v_h, const msa_bf16 *q_idx_h, const msa_bf16 *k_idx_h,
                     msa_bf16 *out_h, float *lse_h, const msa_staging *dev, void *ws,
                     size_t ws_bytes, msa_stream stream, msa_stream copy_stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q_h || !k_h || !v_h || !q_idx_h || !k_idx_h || !out_h || !dev)
    return fail(MSA_ERR_INVALID_ARG, "NULL host pointer or staging");
  if (!dev->q || !dev->k || !dev->v || !dev->q_idx || !dev->k_idx || !dev->out ||
      (lse_h && !dev->lse))
    return fail(MSA_ERR_INVALID_ARG, "NULL staging pointer");
  if (!aligned16(dev->q) || !aligned16(dev->k) || !aligned16(dev->v) || !aligned16(dev->q_idx) ||
      !aligned16(dev->k_idx) || !aligned16(dev->out) || (dev->lse && !aligned16(dev->lse)))
    return fail(MSA_ERR_INVALID_ARG, "staging pointers must be 16-byte aligned");
  const size_t base = msa::kWsHeader + forward_sel_bytes(p);
  rc = check_ws(ws, ws_bytes, attn_ws(p, base).end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t cp = reinterpret_cast<cudaStream_t>(copy_stream);

  std::lock_guard<std::mutex> lock(g_host_mu);
  HostEvents *ev = nullptr;
  rc = host_events(&ev);
  if (rc) return rc;
  AttnPlan pl;
  rc = plan_attn(p, dev->k, dev->v, base, whole(p), &pl);
  if (rc) return rc;
  int32_t *sel = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + msa::kWsHeader);
  const ChunkSink sink{ev->down, ev->chunk, out_h, lse_h};
  // Per query chunk [t0, t0+Lc): upload the chunk's rows (index inputs
  // first), run the index branch for the chunk's query tiles and the main
  // branch for its queries, download its output.  A chunk only needs rows
  // < t0 + Lc, so uploads, computation and downloads of neighbouring chunks
  // overlap; uploads run ahead on copy_stream, downloads on the library's
  // download stream.
  for (int t0 = 0; t0 < p->L; t0 += pl.w.Lc) {
    const int Lc = (p->L - t0) < pl.w.Lc ? (p->L - t0) : pl.w.Lc;
    cudaError_t e = cudaSuccess;
    auto up = [&](msa_bf16 *d, const msa_bf16 *h, size_t row) {   // rows [t0, t0+Lc) of each b
      for (int b = 0; b < p->B && e == cudaSuccess; ++b) {
        const size_t off = (size_t(b) * p->L + t0) * row;
        e = cudaMemcpyAsync(d + off, h + off, size_t(Lc) * row * 2, cudaMemcpyHostToDevice, cp);
      }
    };
    up(dev->k_idx, k_idx_h, size_t(p->d_idx));
    up(dev->q_idx, q_idx_h, size_t(p->G) * p->d_idx);
    if (e == cudaSuccess) e = cudaEventRecord(ev->idx_in, cp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev->idx_in, 0);
    if (e != cudaSuccess) return cuda_fail(e, "index input upload");
    rc = run_index_select(p, dev->q_idx, dev->k_idx, sel, nullptr, ws, st, whole(p), t0, t0 + Lc);
    if (rc) return rc;
    up(dev->k, k_h, size_t(p->G) * p->d);
    up(dev->v, v_h, size_t(p->G) * p->d);
    up(dev->q, q_h, size_t(p->H) * p->d);
    if (e == cudaSuccess) e = cudaEventRecord(ev->all_in, cp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev->all_in, 0);
    if (e != cudaSuccess) return cuda_fail(e, "main input upload");
    rc = run_attn_chunk(p, pl, dev->q, sel, dev->out, lse_h ? dev->lse : nullptr, ws, t0, Lc, st,
                        &sink);
    if (rc) return rc;
  }
  cudaError_t e = cudaSuccess;
  // later work on `stream` runs after the last download
  e = cudaEventRecord(ev->done, ev->down);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev->done, 0);
  if (e != cudaSuccess) return cuda_fail(e, "download completion");
  return MSA_OK;
}

int msa_sparse_attn_backward(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k,
                             const msa_bf16 *v, const msa_bf16 *out, const float *lse,
                             const msa_bf16 *dout, const int32_t *sel, msa_bf16 *dq,
                             msa_bf16 *dk, msa_bf16 *dv, void *ws, size_t ws_bytes,
                             msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k || !v || !out || !lse || !dout || !sel || !dq || !dk || !dv)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(sel) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const BwdWs w = bwd_ws(p);
  const size_t entries = size_t(p->B) * p->G * w.Lc * p->top_k;
  if (entries * (p->H / p->G) >= (size_t(1) << 31))
    return fail(MSA_ERR_UNSUPPORTED, "B*chunk*H*top_k = %zu partial rows (limit 2^31)",
                entries * (p->H / p->G));
  rc = check_ws(ws, ws_bytes, w.end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  const int nb = p->L / 128;
  CUtensorMap tk, tv;
  {
    const uint64_t dims[3] = {uint64_t(p->d), uint64_t(p->G), uint64_t(p->B) * p->L};
    const uint64_t str[2] = {uint64_t(p->d) * 2, uint64_t(p->d) * 2 * p->G};
    const uint32_t box[3] = {64, 1, 128};
    rc = make_tmap(&tk, k, 3, dims, str, box);
    if (rc) return rc;
    rc = make_tmap(&tv, v, 3, dims, str, box);
    if (rc) return rc;
  }
  msa::RevIdxArgs ra;
  ra.B = p->B; ra.G = p->G; ra.L = p->L; ra.nb = nb; ra.top_k = p->top_k;
  ra.qpi = 128 / (p->H / p->G);
  ra.Lq = p->L; ra.tq0 = 0;
  ra.sel = sel;
  ra.cnt = reinterpret_cast<int32_t *>(wsb + w.cnt);
  ra.list_off = reinterpret_cast<int32_t *>(wsb + w.list_off);
  ra.item_off = reinterpret_cast<int32_t *>(wsb + w.item_off);
  ra.list = reinterpret_cast<int32_t *>(wsb + w.list);
  ra.pos_of = reinterpret_cast<int32_t *>(wsb + w.pos_of);
  ra.status = status_ptr(ws);
  msa::BwdArgs a;
  a.B = p->B; a.L = p->L; a.H = p->H; a.G = p->G; a.nb = nb; a.top_k = p->top_k;
  a.scale = eff_scale(p);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.q = q; a.out = out; a.dout = dout; a.lse = lse; a.sel = sel;
  a.list = ra.list; a.list_off = ra.list_off; a.pos_of = ra.pos_of;
  a.delta = reinterpret_cast<float *>(wsb + w.delta);
  a.part_dq = reinterpret_cast<uint16_t *>(wsb + w.part_dq);
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.acc_dk = w.acc_dk ? reinterpret_cast<float *>(wsb + w.acc_dk) : nullptr;
  a.acc_dv = w.acc_dv ? reinterpret_cast<float *>(wsb + w.acc_dv) : nullptr;
  a.unit_ctr = reinterpret_cast<int *>(wsb + 16);
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_bwd_delta(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward D launch");
  if (a.acc_dk) {
    e = cudaMemsetAsync(wsb + w.acc_dk, 0, w.acc_dv - w.acc_dk, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(wsb + w.acc_dv, 0, w.end - w.acc_dv, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward accumulator reset");
  }
  const int sms = num_sms();
  for (int t0 = 0; t0 < p->L; t0 += w.Lc) {
    const int Lc = (p->L - t0) < w.Lc ? (p->L - t0) : w.Lc;
    ra.t0 = t0; ra.Lc = Lc;
    e = msa::launch_revidx(ra, st);
    if (e != cudaSuccess) return cuda_fail(e, "reverse index launch");
    a.t0 = t0; a.Lc = Lc;
    a.last = (t0 + Lc >= p->L) ? 1 : 0;
    e = msa::launch_backward(tk, tv, a, sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  }
  return MSA_OK;
}

int msa_sparse_attn_decode(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                           const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                           const msa_bf16 *k_idx_cache, const int32_t *seq_lens, msa_bf16 *out,
                           int32_t *sel, void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  return run_decode(p, q, q_idx, k_cache, v_cache, k_idx_cache, Fp8Caches{}, seq_lens, out, sel,
                    ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int msa_sparse_attn_decode_fp8idx(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                                  const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                                  const uint8_t *k_idx8, const float *k_idx_scale,
                                  const int32_t *seq_lens, msa_bf16 *out, int32_t *sel, void *ws,
                                  size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  if (!k_idx8) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  Fp8Caches f8;
  f8.k_idx8 = k_idx8;
  f8.k_idx_scale = k_idx_scale;
  return run_decode(p, q, q_idx, k_cache, v_cache, nullptr, f8, seq_lens, out, sel, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

int msa_sparse_attn_decode_fp8(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                               const uint8_t *k8, const float *k_scale, const uint8_t *v8,
                               const float *v_scale, const uint8_t *k_idx8,
                               const float *k_idx_scale, const int32_t *seq_lens, msa_bf16 *out,
                               int32_t *sel, void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  if (!k_idx8 || !k8) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  Fp8Caches f8;
  f8.k_idx8 = k_idx8;
  f8.k_idx_scale = k_idx_scale;
  f8.k8 = k8;
  f8.v8 = v8;
  f8.k_scale = k_scale;
  f8.v_scale = v_scale;
  return run_decode(p, q, q_idx, nullptr, nullptr, nullptr, f8, seq_lens, out, sel, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

int msa_quantize_e4m3_rows(const msa_bf16 *x, long long rows, int cols, uint8_t *codes,
                           float *scale, msa_stream stream) {
  g_err[0] = 0;
  if (rows < 0 || cols <= 0 || cols % 16 != 0)
    return fail(MSA_ERR_INVALID_ARG, "rows=%lld cols=%d: cols must be a positive multiple of 16",
                rows, cols);
  if (rows == 0) return MSA_OK;
  if (!x || !codes || !scale) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scale))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  cudaError_t e = msa::launch_quantize_e4m3_rows(x, rows, cols, codes, scale,
                                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return MSA_OK;
}

}  // extern "C"
