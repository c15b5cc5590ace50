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
#include <algorithm>
#include <mutex>
#include <vector>

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
// Every operation takes any sequence length and either block length.
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
  if (p->block != 128 && p->block != 64)
    return fail(MSA_ERR_UNSUPPORTED, "block=%d (supported: 64, 128)", p->block);
  if (p->top_k > msa::kMaxTopK)
    return fail(MSA_ERR_UNSUPPORTED, "top_k=%d (supported: 1..32)", p->top_k);
  if (p->H % p->G != 0) return fail(MSA_ERR_INVALID_ARG, "H=%d not a multiple of G=%d", p->H, p->G);
  const int r = p->H / p->G;
  if (r != 1 && r != 2 && r != 4 && r != 8 && r != 16)
    return fail(MSA_ERR_UNSUPPORTED, "H/G=%d (supported: 1,2,4,8,16)", r);
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

// Key blocks of a sequence of L tokens (the last one may be partial).
int nblocks(const msa_params *p, int L) { return (L + p->block - 1) / p->block; }
int nblocks(const msa_params *p) { return nblocks(p, p->L); }

// ---- workspace plans --------------------------------------------------------
// Prefill attention processes the packed query rows in chunks of Rc so that
// the partial results (bf16, one 128-wide row per selected (query, head,
// slot)) stay within a fixed budget.  Every chunk reads the K/V blocks its
// queries select, which for long inputs is most of K/V, so fewer, larger
// chunks cut K/V re-reads: 16 GiB of partials is 9 chunks at 1M tokens,
// H=32, top_k=16 (a small share of HBM on this part).
constexpr size_t kPartialBudget = size_t(16) << 30;  // 16 GiB

int prefill_chunk(const msa_params *p, long long n_rows) {
  const size_t per_row = size_t(p->H) * p->top_k * (p->d * 2 + 4);
  long long rc = (long long)(kPartialBudget / per_row);
  rc = (rc / 128) * 128;
  if (rc < 128) rc = 128;
  if (p->chunk > 0 && p->chunk < rc) rc = p->chunk;
  if (rc > n_rows) rc = n_rows;
  return (int)rc;
}

struct AttnWs {
  size_t cnt, list_off, item_off, list, pos_of, part_o, part_lse, end;
  int Rc;
};
// n_rows packed query rows of n_seq sequences of up to p->L keys each.
AttnWs attn_ws(const msa_params *p, size_t base, long long n_rows, int n_seq) {
  AttnWs w;
  w.Rc = prefill_chunk(p, n_rows);
  const size_t nbgj = size_t(n_seq) * p->G * nblocks(p);
  const size_t entries = size_t(p->G) * w.Rc * p->top_k;
  size_t o = base;
  w.cnt = o; o = align_up(o + 4 * nbgj);
  w.list_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.item_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.list = o; o = align_up(o + 4 * entries);
  w.pos_of = o; o = align_up(o + 4 * entries);
  w.part_o = o; o = align_up(o + 2 * entries * (p->H / p->G) * size_t(p->d));
  w.part_lse = o; o = align_up(o + 4 * entries * (p->H / p->G));
  w.end = o;
  return w;
}
AttnWs attn_ws(const msa_params *p, size_t base) {
  return attn_ws(p, base, (long long)p->B * p->L, p->B);
}

// Backward: D = do . o per row; per query chunk (the prefill's chunk length,
// packed rows b*L + t) a reverse index and one bf16 dq partial row per
// (query, head, slot); with more than one chunk, fp32 dk/dv accumulators
// over the whole batch.
struct BwdWs {
  size_t cnt, list_off, item_off, list, pos_of, delta, part_dq, acc_dk, acc_dv, end;
  int Rc;
};
// At most 2^19 rows per chunk: the reverse index's ordering step keeps a
// bitmap of one sequence's rows in a chunk, and its prefix counts, in
// shared memory (128 KiB at that bound).
constexpr int kBwdMaxChunkRows = 1 << 19;
BwdWs bwd_ws(const msa_params *p) {
  BwdWs w;
  const long long n_rows = (long long)p->B * p->L;
  w.Rc = prefill_chunk(p, n_rows);
  if (w.Rc > kBwdMaxChunkRows) w.Rc = kBwdMaxChunkRows;
  const size_t nbgj = size_t(p->B) * p->G * nblocks(p);
  const size_t entries = size_t(p->G) * w.Rc * p->top_k;
  size_t o = msa::kWsHeader;
  w.cnt = o; o = align_up(o + 4 * nbgj);
  w.list_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.item_off = o; o = align_up(o + 4 * (nbgj + 1));
  w.list = o; o = align_up(o + 4 * entries);
  w.pos_of = o; o = align_up(o + 4 * entries);
  w.delta = o; o = align_up(o + 4 * size_t(n_rows) * p->H);
  w.part_dq = o; o = align_up(o + 2 * entries * (p->H / p->G) * size_t(p->d));
  w.acc_dk = w.acc_dv = 0;
  if (w.Rc < n_rows) {
    const size_t kv = 4 * size_t(n_rows) * p->G * p->d;
    w.acc_dk = o; o = align_up(o + kv);
    w.acc_dv = o; o = align_up(o + kv);
  }
  w.end = o;
  return w;
}

struct DecWs {
  size_t scores, sel, part_o, part_lse, tickets, end;
};
DecWs dec_ws(const msa_params *p) {
  DecWs w;
  const size_t nb = size_t(nblocks(p));
  size_t o = msa::kWsHeader;
  w.scores = o; o = align_up(o + 4 * size_t(p->B) * p->G * nb);
  w.sel = o; o = align_up(o + 4 * size_t(p->B) * p->G * p->top_k);
  w.part_o = o; o = align_up(o + 4 * size_t(p->B) * p->H * p->top_k * p->d);
  w.part_lse = o; o = align_up(o + 4 * size_t(p->B) * p->H * p->top_k);
  w.tickets = o; o = align_up(o + 4 * size_t(p->B) * p->G);
  w.end = o;
  return w;
}

size_t forward_sel_bytes(const msa_params *p) {
  return align_up(4 * size_t(p->B) * p->G * p->L * p->top_k);
}

// Ragged batch (msa_forward_cached_varlen): device tables at the start of
// the workspace, after the header -- two 4-D K/V tensor maps per sequence,
// the per-sequence query geometry, and the index branch's (b, tile) list --
// then the selection of the packed rows, then the attention workspace.
struct VarlenWs {
  size_t maps, seqs, items, sel, attn_base;
};
VarlenWs varlen_ws(const msa_params *p) {
  VarlenWs w;
  size_t o = msa::kWsHeader;
  w.maps = o; o = align_up(o + 2 * sizeof(CUtensorMap) * size_t(p->B));
  w.seqs = o; o = align_up(o + sizeof(int4) * size_t(p->B));
  w.items = o; o = align_up(o + sizeof(int2) * size_t(p->B) * ((p->L + 127) / 128));   // query tiles
  w.sel = o; o += forward_sel_bytes(p);
  w.attn_base = o;
  return w;
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
// Elements outside the dims load as zeros.
int make_tmap(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
              const uint64_t *strides_bytes, const uint32_t *box) {
  auto fn = encode_fn();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  uint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
                  strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MSA_OK;
}

// 4-D map (d, G, key rows, sequences) over K or V [nseq, L, G, d], the row
// extent cut at kv_rows: rows >= kv_rows of each sequence load as zeros.
// A box is one block of keys (p->block rows) of one KV head, half of d.
int make_kv_tmap(CUtensorMap *m, const void *base, const msa_params *p, int kv_rows, int nseq) {
  const uint64_t dims[4] = {uint64_t(p->d), uint64_t(p->G), uint64_t(kv_rows), uint64_t(nseq)};
  const uint64_t str[3] = {uint64_t(p->d) * 2, uint64_t(p->d) * 2 * p->G,
                           uint64_t(p->d) * 2 * p->G * p->L};
  const uint32_t box[4] = {64, 1, uint32_t(p->block), 1};
  return make_tmap(m, base, 4, dims, str, box);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int *status_ptr(void *ws) { return reinterpret_cast<int *>(ws); }

// ---- the operations --------------------------------------------------------
// Query-side geometry of a uniform batch: every sequence has Lq query rows at
// positions [tq0, tq0 + Lq) (see msa::QGeo).
msa::QGeo uniform_geo(const msa_params *p, int Lq, int tq0) {
  msa::QGeo q;
  q.seqs = nullptr;
  q.B = p->B; q.G = p->G; q.Lq = Lq; q.tq0 = tq0;
  q.N = p->B * Lq;
  q.sel_gs = Lq;
  return q;
}
msa::QGeo whole(const msa_params *p) { return uniform_geo(p, p->L, 0); }

// Which index work a launch does and which rows it writes.
struct IndexWork {
  int i_hi = 0, n_tiles = 0;        // uniform: tiles [i_hi - n_tiles, i_hi) of every sequence
  const int2 *items = nullptr;      // ragged: (b, tile) pairs in device memory
  int n_tab = 0;
  int r_lo = 0, r_hi = 0;           // packed rows written
};

// Uniform work: the tiles covering positions [t_lo, t_hi) of every sequence,
// writing the packed rows of those positions.
IndexWork uniform_index_work(const msa::QGeo &q, int t_lo, int t_hi) {
  IndexWork w;
  w.i_hi = (t_hi + 127) / 128;
  w.n_tiles = w.i_hi - t_lo / 128;
  if (q.B == 1) {
    w.r_lo = t_lo - q.tq0;
    w.r_hi = t_hi - q.tq0;
  } else {   // whole sequences
    w.r_lo = 0;
    w.r_hi = q.N;
  }
  return w;
}

int run_index_select(const msa_params *p, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                     int32_t *sel, float *block_scores, void *ws, cudaStream_t st,
                     const msa::QGeo &qg, const IndexWork &iw) {
  const int nb = nblocks(p);
  CUtensorMap tq, tk;
  {
    const uint64_t dims[3] = {uint64_t(p->d_idx), uint64_t(p->G), uint64_t(qg.N)};
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
  a.blk = p->block;
  a.q = qg;
  a.write_scores = block_scores ? 1 : 0;
  a.i_hi = iw.i_hi;
  a.n_tiles = iw.n_tiles;
  a.items = iw.items;
  const int ngp = p->G / msa::index_groups_per_cta(p->G, p->top_k);
  a.n_items = (iw.items ? iw.n_tab : p->B * iw.n_tiles) * ngp;
  a.r_lo = iw.r_lo;
  a.r_hi = iw.r_hi;
  a.sel = sel;
  a.scores = block_scores;
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_index_kernel(tq, tk, a, num_sms(), st);
  if (e != cudaSuccess) return cuda_fail(e, "index kernel launch");
  if (block_scores) {
    msa::TopkArgs t;
    t.B = p->B; t.G = p->G; t.L = p->L; t.nb = nb; t.top_k = p->top_k; t.blk = p->block;
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
  CUtensorMap tk, tv;               // launch maps (uniform batch)
  const CUtensorMap *kv_maps;       // per-sequence maps in device memory (ragged), or null
  AttnWs w;
  int nb, qpi, sms;
  float scale;
  msa::QGeo qg;
};

// kv_rows: key rows every sequence may attend (uniform batch; rows past it
// load as zeros); kv_maps: per-sequence maps instead (ragged batch).
int plan_attn(const msa_params *p, const msa_bf16 *k, const msa_bf16 *v, size_t ws_base,
              const msa::QGeo &qg, int kv_rows, const CUtensorMap *kv_maps, AttnPlan *pl) {
  pl->nb = nblocks(p);
  pl->qg = qg;
  pl->kv_maps = kv_maps;
  pl->w = attn_ws(p, ws_base, qg.N, qg.B);
  int rc = make_kv_tmap(&pl->tk, k, p, kv_rows, p->B);
  if (rc) return rc;
  rc = make_kv_tmap(&pl->tv, v, p, kv_rows, p->B);
  if (rc) return rc;
  pl->qpi = 128 / (p->H / p->G);
  pl->scale = eff_scale(p);
  pl->sms = num_sms();
  return MSA_OK;
}

// One query chunk, packed rows [r0, r0 + Rc): reverse index, attention,
// merge; then, with a sink, the download of the chunk's output rows.
int run_attn_chunk(const msa_params *p, const AttnPlan &pl, const msa_bf16 *q, const int32_t *sel,
                   msa_bf16 *out, float *lse, void *ws, int r0, int Rc, cudaStream_t st,
                   const ChunkSink *sink) {
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  const AttnWs &w = pl.w;
  msa::RevIdxArgs ra;
  ra.G = p->G; ra.nb = pl.nb; ra.top_k = p->top_k; ra.qpi = pl.qpi;
  ra.q = pl.qg;
  ra.order_words = 0;   // attention partials are merged in slot order: any list order
  ra.r0 = r0; ra.Rc = Rc;
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
  aa.L = p->L; aa.H = p->H; aa.G = p->G; aa.nb = pl.nb; aa.top_k = p->top_k;
  aa.blk = p->block;
  aa.q = pl.qg;
  aa.scale = pl.scale;
  aa.scale_log2 = pl.scale * 1.4426950408889634f;
  const long long max_items =
      (long long)p->G * Rc * p->top_k / pl.qpi + (long long)pl.qg.B * p->G * pl.nb;
  aa.max_items = (int)max_items;
  aa.q_ptr = q;
  aa.kv_maps = pl.kv_maps;
  aa.list = ra.list; aa.list_off = ra.list_off; aa.item_off = ra.item_off;
  aa.part_o = reinterpret_cast<uint16_t *>(wsb + w.part_o);
  aa.part_lse = reinterpret_cast<float *>(wsb + w.part_lse);
  aa.status = status_ptr(ws);
  e = msa::launch_prefill_attn(pl.tk, pl.tv, aa, pl.sms, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
  msa::CombineArgs ca;
  ca.H = p->H; ca.G = p->G; ca.top_k = p->top_k;
  ca.q = pl.qg;
  ca.r0 = r0; ca.Rc = Rc;
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
    const size_t row = size_t(p->H) * p->d;   // elements of one query row's output
    e = cudaMemcpyAsync(sink->out_h + size_t(r0) * row, out + size_t(r0) * row,
                        size_t(Rc) * row * 2, cudaMemcpyDeviceToHost, sink->copy);
    if (e == cudaSuccess && sink->lse_h)
      e = cudaMemcpyAsync(sink->lse_h + size_t(r0) * p->H, lse + size_t(r0) * p->H,
                          size_t(Rc) * p->H * 4, cudaMemcpyDeviceToHost, sink->copy);
    if (e != cudaSuccess) return cuda_fail(e, "output download");
  }
  return MSA_OK;
}

// Main branch for every packed query row of the plan.
int run_prefill_attn(const msa_params *p, const AttnPlan &pl, const msa_bf16 *q,
                     const int32_t *sel, msa_bf16 *out, float *lse, void *ws, cudaStream_t st) {
  for (int r0 = 0; r0 < pl.qg.N; r0 += pl.w.Rc) {
    const int Rc = (pl.qg.N - r0) < pl.w.Rc ? (pl.qg.N - r0) : pl.w.Rc;
    const int rc = run_attn_chunk(p, pl, q, sel, out, lse, ws, r0, Rc, st, nullptr);
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
  a.nb_max = nblocks(p); a.top_k = p->top_k;
  a.blk = p->block;
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
  a.tickets = reinterpret_cast<int *>(wsb + w.tickets);
  a.out = out;
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_decode(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return MSA_OK;
}

// ---- NSA-style branches ------------------------------------------------------
// Workspace of msa_nsa_forward: msa_forward's, then the compressed keys and
// values and the compression and window branches' outputs.
struct NsaWs {
  size_t fwd_end, k_cmp, v_cmp, o_cmp, o_win, end;
};
NsaWs nsa_ws(const msa_params *p) {
  NsaWs w;
  w.fwd_end = attn_ws(p, msa::kWsHeader + forward_sel_bytes(p)).end;
  const size_t cmp = align_up(2 * size_t(p->B) * nblocks(p) * p->G * p->d);
  const size_t o = align_up(2 * size_t(p->B) * p->L * p->H * p->d);
  size_t x = align_up(w.fwd_end);
  w.k_cmp = x; x += cmp;
  w.v_cmp = x; x += cmp;
  w.o_cmp = x; x += o;
  w.o_win = x; x += o;
  w.end = x;
  return w;
}

// 4-D map over q [B,L,H,d] as (d, H, L, B): a box is 128/R consecutive
// queries x the R heads of one group (a 128-row tile), half of d.
int make_q_tmap(CUtensorMap *m, const void *q, const msa_params *p) {
  const int r = p->H / p->G;
  const uint64_t dims[4] = {uint64_t(p->d), uint64_t(p->H), uint64_t(p->L), uint64_t(p->B)};
  const uint64_t str[3] = {uint64_t(p->d) * 2, uint64_t(p->d) * 2 * p->H,
                           uint64_t(p->d) * 2 * p->H * p->L};
  const uint32_t box[4] = {64, uint32_t(r), uint32_t(128 / r), 1};
  return make_tmap(m, q, 4, dims, str, box);
}

// 4-D map over key rows [B, rows, G, d] as (d, G, rows, B): a box is 128
// rows of one KV head, half of d; rows past `rows` load as zeros.
int make_rows_tmap(CUtensorMap *m, const void *base, const msa_params *p, int rows) {
  const uint64_t dims[4] = {uint64_t(p->d), uint64_t(p->G), uint64_t(rows), uint64_t(p->B)};
  const uint64_t str[3] = {uint64_t(p->d) * 2, uint64_t(p->d) * 2 * p->G,
                           uint64_t(p->d) * 2 * p->G * rows};
  const uint32_t box[4] = {64, 1, 128, 1};
  return make_tmap(m, base, 4, dims, str, box);
}

// One branch: mode 0 = window over the tokens k, v [B,L,G,d]; mode 1 =
// compressed tokens k, v [B,nb,G,d].
int run_dense(const msa_params *p, int mode, int window, const msa_bf16 *q, const void *k,
              const void *v, int rows, msa_bf16 *out, float *lse, void *ws, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  int rc = make_q_tmap(&tq, q, p);
  if (rc) return rc;
  rc = make_rows_tmap(&tk, k, p, rows);
  if (rc) return rc;
  rc = make_rows_tmap(&tv, v, p, rows);
  if (rc) return rc;
  msa::DenseAttnArgs a;
  a.B = p->B; a.L = p->L; a.H = p->H; a.G = p->G;
  const int qpi = 128 / (p->H / p->G);
  a.n_qt = (p->L + qpi - 1) / qpi;
  a.mode = mode; a.window = window; a.blk = p->block;
  a.scale = eff_scale(p);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.out = reinterpret_cast<uint16_t *>(out);
  a.lse = lse;
  a.status = status_ptr(ws);
  cudaError_t e = msa::launch_dense_attn(tq, tk, tv, a, num_sms(), st);
  if (e != cudaSuccess) return cuda_fail(e, "NSA branch attention launch");
  return MSA_OK;
}

int nsa_compress(const msa_params *p, const msa_bf16 *k, const msa_bf16 *v, msa_bf16 *k_cmp,
                 msa_bf16 *v_cmp, cudaStream_t st) {
  cudaError_t e = msa::launch_nsa_compress(k, v, k_cmp, v_cmp, p->B, p->L, p->G, p->block, st);
  if (e != cudaSuccess) return cuda_fail(e, "NSA compression launch");
  return MSA_OK;
}

int nsa_gate(const msa_params *p, const float *gates, const msa_bf16 *o_cmp, const msa_bf16 *o_slc,
             const msa_bf16 *o_win, msa_bf16 *out, cudaStream_t st) {
  cudaError_t e = msa::launch_nsa_gate(gates, o_cmp, o_slc, o_win, out,
                                       (long long)p->B * p->L * p->H, st);
  if (e != cudaSuccess) return cuda_fail(e, "NSA gate launch");
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
    case MSA_OP_FORWARD_VARLEN: return attn_ws(p, varlen_ws(p).attn_base).end;
    case MSA_OP_NSA_BRANCH: return msa::kWsHeader;
    case MSA_OP_NSA_FORWARD: return nsa_ws(p).end;
    default: fail(MSA_ERR_INVALID_ARG, "unknown op %d", op); return 0;
  }
}

int msa_prefill_chunk_len(const msa_params *p) {
  g_err[0] = 0;
  if (check_params(p, false) != MSA_OK) return 0;
  return p->L > 0 && p->B > 0 ? prefill_chunk(p, (long long)p->B * p->L) : 0;
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
  const msa::QGeo qg = whole(p);
  return run_index_select(p, q_idx, k_idx, sel, block_scores, ws,
                          reinterpret_cast<cudaStream_t>(stream), qg,
                          uniform_index_work(qg, 0, p->L));
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
  rc = check_ws(ws, ws_bytes, attn_ws(p, msa::kWsHeader).end);
  if (rc) return rc;
  AttnPlan pl;
  rc = plan_attn(p, k, v, msa::kWsHeader, whole(p), p->L, nullptr, &pl);
  if (rc) return rc;
  return run_prefill_attn(p, pl, q, sel, out, lse, ws, reinterpret_cast<cudaStream_t>(stream));
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
  const msa::QGeo qg = whole(p);
  rc = run_index_select(p, q_idx, k_idx, s, nullptr, ws, st, qg, uniform_index_work(qg, 0, p->L));
  if (rc) return rc;
  AttnPlan pl;
  rc = plan_attn(p, k, v, base, qg, p->L, nullptr, &pl);
  if (rc) return rc;
  return run_prefill_attn(p, pl, q, s, out, lse, ws, st);
}

int msa_forward_cached(const msa_params *p, int t0, int n, const msa_bf16 *q,
                       const msa_bf16 *q_idx, const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                       const msa_bf16 *k_idx_cache, msa_bf16 *out, int32_t *sel, float *lse,
                       void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (t0 < 0 || n < 0 || (long long)t0 + n > p->L)
    return fail(MSA_ERR_INVALID_ARG, "t0=%d n=%d: need t0, n >= 0 and t0 + n <= L=%d", t0, n, p->L);
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
  const msa::QGeo qg = uniform_geo(p, n, t0);
  int32_t *s = sel ? sel : reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + msa::kWsHeader);
  IndexWork iw = uniform_index_work(qg, t0, t0 + n);
  iw.r_lo = 0;
  iw.r_hi = qg.N;
  rc = run_index_select(p, q_idx, k_idx_cache, s, nullptr, ws, st, qg, iw);
  if (rc) return rc;
  AttnPlan pl;
  rc = plan_attn(p, k_cache, v_cache, base, qg, t0 + n, nullptr, &pl);
  if (rc) return rc;
  return run_prefill_attn(p, pl, q, s, out, lse, ws, st);
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
  long long N = 0;
  for (int b = 0; b < p->B; ++b) {
    if (t0[b] < 0 || n[b] < 0 || (long long)t0[b] + n[b] > p->L)
      return fail(MSA_ERR_INVALID_ARG, "sequence %d: t0=%d n=%d (need t0, n >= 0, t0+n <= L=%d)",
                  b, t0[b], n[b], p->L);
    N += n[b];
  }
  if (N == 0) return MSA_OK;
  if (!q || !q_idx || !k_cache || !v_cache || !k_idx_cache || !out)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(q_idx) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(k_idx_cache) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const VarlenWs vw = varlen_ws(p);
  rc = check_ws(ws, ws_bytes, attn_ws(p, vw.attn_base).end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);

  // Host-built tables: per-sequence K/V maps (row extent t0 + n, so keys past
  // a sequence's end load as zeros), query geometry, and the index branch's
  // (b, tile) work list, longest tiles first.
  const int B = p->B;
  std::vector<uint8_t> tab(vw.sel - vw.maps, 0);
  CUtensorMap *maps = reinterpret_cast<CUtensorMap *>(tab.data());
  int4 *seqs = reinterpret_cast<int4 *>(tab.data() + (vw.seqs - vw.maps));
  int2 *items = reinterpret_cast<int2 *>(tab.data() + (vw.items - vw.maps));
  const size_t kv_seq = size_t(p->L) * p->G * p->d;   // elements per sequence
  int row0 = 0, n_tab = 0;
  for (int b = 0; b < B; ++b) {
    const int kv_rows = t0[b] + n[b] > 0 ? t0[b] + n[b] : 1;
    rc = make_kv_tmap(&maps[2 * b], k_cache + b * kv_seq, p, kv_rows, 1);
    if (rc) return rc;
    rc = make_kv_tmap(&maps[2 * b + 1], v_cache + b * kv_seq, p, kv_rows, 1);
    if (rc) return rc;
    seqs[b] = make_int4(row0, t0[b], n[b], row0);
    if (n[b] > 0)
      for (int i = t0[b] / 128; i < (t0[b] + n[b] + 127) / 128; ++i) items[n_tab++] = make_int2(b, i);
    row0 += n[b];
  }
  std::stable_sort(items, items + n_tab, [](const int2 &x, const int2 &y) { return x.y > y.y; });
  const size_t tab_bytes = (vw.items - vw.maps) + sizeof(int2) * size_t(n_tab);
  cudaError_t e = cudaMemcpyAsync(wsb + vw.maps, tab.data(), tab_bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "ragged batch tables upload");

  msa::QGeo qg;
  qg.seqs = reinterpret_cast<const int4 *>(wsb + vw.seqs);
  qg.B = B; qg.G = p->G; qg.Lq = 0; qg.tq0 = 0;
  qg.N = (int)N;
  qg.sel_gs = (int)N;
  int32_t *sel = reinterpret_cast<int32_t *>(wsb + vw.sel);
  IndexWork iw;
  iw.items = reinterpret_cast<const int2 *>(wsb + vw.items);
  iw.n_tab = n_tab;
  iw.r_lo = 0;
  iw.r_hi = (int)N;
  rc = run_index_select(p, q_idx, k_idx_cache, sel, nullptr, ws, st, qg, iw);
  if (rc) return rc;
  AttnPlan pl;
  rc = plan_attn(p, k_cache, v_cache, vw.attn_base, qg, p->L,
                 reinterpret_cast<const CUtensorMap *>(wsb + vw.maps), &pl);
  if (rc) return rc;
  return run_prefill_attn(p, pl, q, sel, out, lse, ws, st);
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
  // One sequence at a time (a B = 1 problem at the sequence's offsets), each
  // pipelined per query chunk [t0, t0+Lc): upload the chunk's rows (index
  // inputs first), run the index branch for the chunk's query tiles and the
  // main branch for its queries, download its output.  A chunk only needs
  // rows < t0 + Lc, so uploads, computation and downloads of neighbouring
  // chunks overlap; uploads run ahead on copy_stream, downloads on the
  // library's download stream.
  msa_params p1 = *p;
  p1.B = 1;
  const msa::QGeo qg = whole(&p1);
  int32_t *sel = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) + msa::kWsHeader);
  for (int b = 0; b < p->B; ++b) {
    const size_t rows0 = size_t(b) * p->L;   // first row of sequence b
    auto at = [&](auto *ptr, size_t row_elems) { return ptr + rows0 * row_elems; };
    const size_t e_q = size_t(p->H) * p->d, e_kv = size_t(p->G) * p->d;
    const size_t e_qi = size_t(p->G) * p->d_idx, e_ki = size_t(p->d_idx);
    AttnPlan pl;
    rc = plan_attn(&p1, at(dev->k, e_kv), at(dev->v, e_kv), base, qg, p->L, nullptr, &pl);
    if (rc) return rc;
    const ChunkSink sink{ev->down, ev->chunk, at(out_h, e_q), lse_h ? at(lse_h, size_t(p->H)) : nullptr};
    for (int t0 = 0; t0 < p->L; t0 += pl.w.Rc) {
      const int Lc = (p->L - t0) < pl.w.Rc ? (p->L - t0) : pl.w.Rc;
      cudaError_t e = cudaSuccess;
      auto up = [&](msa_bf16 *d, const msa_bf16 *h, size_t row) {   // rows [t0, t0+Lc)
        if (e != cudaSuccess) return;
        const size_t off = (rows0 + t0) * row;
        e = cudaMemcpyAsync(d + off, h + off, size_t(Lc) * row * 2, cudaMemcpyHostToDevice, cp);
      };
      up(dev->k_idx, k_idx_h, e_ki);
      up(dev->q_idx, q_idx_h, e_qi);
      if (e == cudaSuccess) e = cudaEventRecord(ev->idx_in, cp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev->idx_in, 0);
      if (e != cudaSuccess) return cuda_fail(e, "index input upload");
      rc = run_index_select(&p1, at(dev->q_idx, e_qi), at(dev->k_idx, e_ki), sel, nullptr, ws, st,
                            qg, uniform_index_work(qg, t0, t0 + Lc));
      if (rc) return rc;
      up(dev->k, k_h, e_kv);
      up(dev->v, v_h, e_kv);
      up(dev->q, q_h, e_q);
      if (e == cudaSuccess) e = cudaEventRecord(ev->all_in, cp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev->all_in, 0);
      if (e != cudaSuccess) return cuda_fail(e, "main input upload");
      rc = run_attn_chunk(&p1, pl, at(dev->q, e_q), sel, at(dev->out, e_q),
                          lse_h ? at(dev->lse, size_t(p->H)) : nullptr, ws, t0, Lc, st, &sink);
      if (rc) return rc;
    }
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
  const size_t entries = size_t(p->G) * w.Rc * p->top_k;
  if (entries * (p->H / p->G) >= (size_t(1) << 31))
    return fail(MSA_ERR_UNSUPPORTED, "chunk*H*top_k = %zu partial rows (limit 2^31)",
                entries * (p->H / p->G));
  rc = check_ws(ws, ws_bytes, w.end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  const int nb = nblocks(p);
  const int N = p->B * p->L;
  CUtensorMap tk, tv;
  rc = make_kv_tmap(&tk, k, p, p->L, p->B);
  if (rc) return rc;
  rc = make_kv_tmap(&tv, v, p, p->L, p->B);
  if (rc) return rc;
  msa::RevIdxArgs ra;
  ra.G = p->G; ra.nb = nb; ra.top_k = p->top_k;
  ra.qpi = 128 / (p->H / p->G);
  ra.q = whole(p);
  ra.sel = sel;
  ra.cnt = reinterpret_cast<int32_t *>(wsb + w.cnt);
  ra.list_off = reinterpret_cast<int32_t *>(wsb + w.list_off);
  ra.item_off = reinterpret_cast<int32_t *>(wsb + w.item_off);
  ra.list = reinterpret_cast<int32_t *>(wsb + w.list);
  ra.pos_of = reinterpret_cast<int32_t *>(wsb + w.pos_of);
  // lists in query order: dk and dv sum a block's items in a fixed order
  ra.order_words = ((w.Rc < p->L ? w.Rc : p->L) + 31) / 32;
  ra.status = status_ptr(ws);
  msa::BwdArgs a;
  a.B = p->B; a.L = p->L; a.H = p->H; a.G = p->G; a.nb = nb; a.top_k = p->top_k;
  a.blk = p->block;
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
  for (int r0 = 0; r0 < N; r0 += w.Rc) {
    const int Rc = (N - r0) < w.Rc ? (N - r0) : w.Rc;
    ra.r0 = r0; ra.Rc = Rc;
    e = msa::launch_revidx(ra, st);
    if (e != cudaSuccess) return cuda_fail(e, "reverse index launch");
    a.r0 = r0; a.Rc = Rc;
    a.last = (r0 + Rc >= N) ? 1 : 0;
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

int msa_nsa_compress_kv(const msa_params *p, const msa_bf16 *k, const msa_bf16 *v,
                        msa_bf16 *k_cmp, msa_bf16 *v_cmp, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!k || !v || !k_cmp || !v_cmp) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cmp) || !aligned16(v_cmp))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return nsa_compress(p, k, v, k_cmp, v_cmp, reinterpret_cast<cudaStream_t>(stream));
}

int msa_nsa_window_attn(const msa_params *p, int32_t window, const msa_bf16 *q,
                        const msa_bf16 *k, const msa_bf16 *v, msa_bf16 *out, float *lse,
                        void *ws, size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (window < 1) return fail(MSA_ERR_INVALID_ARG, "window=%d must be >= 1", window);
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k || !v || !out) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  rc = check_ws(ws, ws_bytes, msa::kWsHeader);
  if (rc) return rc;
  return run_dense(p, 0, window, q, k, v, p->L, out, lse, ws,
                   reinterpret_cast<cudaStream_t>(stream));
}

int msa_nsa_compressed_attn(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k_cmp,
                            const msa_bf16 *v_cmp, msa_bf16 *out, float *lse, void *ws,
                            size_t ws_bytes, msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k_cmp || !v_cmp || !out) return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k_cmp) || !aligned16(v_cmp) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  rc = check_ws(ws, ws_bytes, msa::kWsHeader);
  if (rc) return rc;
  return run_dense(p, 1, 0, q, k_cmp, v_cmp, nblocks(p), out, lse, ws,
                   reinterpret_cast<cudaStream_t>(stream));
}

int msa_nsa_gate(const msa_params *p, const float *gates, const msa_bf16 *o_cmp,
                 const msa_bf16 *o_slc, const msa_bf16 *o_win, msa_bf16 *out,
                 msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!gates || !o_cmp || !o_slc || !o_win || !out)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(gates) || !aligned16(o_cmp) || !aligned16(o_slc) || !aligned16(o_win) ||
      !aligned16(out))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return nsa_gate(p, gates, o_cmp, o_slc, o_win, out, reinterpret_cast<cudaStream_t>(stream));
}

int msa_nsa_forward(const msa_params *p, int32_t window, const msa_bf16 *q, const msa_bf16 *k,
                    const msa_bf16 *v, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                    const float *gates, msa_bf16 *out, int32_t *sel, void *ws, size_t ws_bytes,
                    msa_stream stream) {
  g_err[0] = 0;
  int rc = check_params(p, false);
  if (rc) return rc;
  if (window < 1) return fail(MSA_ERR_INVALID_ARG, "window=%d must be >= 1", window);
  if (p->B == 0 || p->L == 0) return MSA_OK;
  if (!q || !k || !v || !q_idx || !k_idx || !gates || !out)
    return fail(MSA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(gates)) return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const NsaWs w = nsa_ws(p);
  rc = check_ws(ws, ws_bytes, w.end);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // selection branch (MSA) into out; its own checks cover q..k_idx, out, sel
  rc = msa_forward(p, q, k, v, q_idx, k_idx, out, sel, nullptr, ws, w.fwd_end, stream);
  if (rc) return rc;
  uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
  msa_bf16 *k_cmp = reinterpret_cast<msa_bf16 *>(wsb + w.k_cmp);
  msa_bf16 *v_cmp = reinterpret_cast<msa_bf16 *>(wsb + w.v_cmp);
  msa_bf16 *o_cmp = reinterpret_cast<msa_bf16 *>(wsb + w.o_cmp);
  msa_bf16 *o_win = reinterpret_cast<msa_bf16 *>(wsb + w.o_win);
  rc = nsa_compress(p, k, v, k_cmp, v_cmp, st);
  if (rc) return rc;
  rc = run_dense(p, 1, 0, q, k_cmp, v_cmp, nblocks(p), o_cmp, nullptr, ws, st);
  if (rc) return rc;
  rc = run_dense(p, 0, window, q, k, v, p->L, o_win, nullptr, ws, st);
  if (rc) return rc;
  return nsa_gate(p, gates, o_cmp, out, o_win, out, st);
}

}  // extern "C"
