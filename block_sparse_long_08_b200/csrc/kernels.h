// Internal launch interface between the C-ABI layer (msa_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace msa {

// Query-side geometry.  Query rows are packed: sequence b owns rows
// [qrow0_b, qrow0_b + nq_b) of q, q_idx, out and lse, holding positions
// [tq0_b, tq0_b + nq_b); its keys are rows [b*L, b*L + tq0_b + nq_b) of k, v
// and k_idx (L = rows per sequence on the key side).  Its selection row for
// group g and position t is sel_base_b + g*sel_gs + (t - tq0_b) (in units of
// top_k entries; block scores use the same row index, in units of nb).
//   uniform batch (seqs == nullptr): qrow0_b = b*Lq, tq0_b = tq0, nq_b = Lq,
//     sel_base_b = b*G*Lq, sel_gs = Lq, N = B*Lq -- the [B,G,Lq,top_k]
//     selection layout of the C ABI;
//   ragged batch: seqs[b] = {qrow0, tq0, nq, sel_base} in device memory
//     (sequences in row order; nq may be 0), sel_gs = N -- a [G,N,top_k]
//     selection over the packed rows.
struct QGeo {
  const int4 *seqs;
  int B, G, Lq, tq0;
  int N;        // packed query rows
  int sel_gs;   // selection rows between groups
};

__device__ __forceinline__ int4 qgeo_seq(const QGeo &q, int b) {
  if (q.seqs) return q.seqs[b];
  return make_int4(b * q.Lq, q.tq0, q.Lq, b * q.G * q.Lq);
}

// Sequence that owns packed row r: the last b with qrow0_b <= r (empty
// sequences share their successor's qrow0 and are skipped that way).
__device__ __forceinline__ int qgeo_seq_of_row(const QGeo &q, int r) {
  if (!q.seqs) return r / q.Lq;
  int lo = 0, hi = q.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q.seqs[mid].x <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Index branch.  Work items are (b, 128-query tile i, group pair): either
// every b with the tiles [i_hi - n_tiles, i_hi), longest first (items ==
// nullptr), or the (b, i) pairs of items[0 .. n_tab) (ragged batches,
// ordered longest first by the host), each with every group pair.
struct IndexArgs {
  int B, L, G, nb, top_k, d_idx;
  int blk;           // block length: 128 or 64 (query tiles are 128 rows either way)
  QGeo q;
  int write_scores;  // 1: store block scores, 0: fused top-k -> sel
  int i_hi, n_tiles; // uniform item range (items == nullptr)
  const int2 *items; // {b, i} pairs (ragged)
  int n_items;       // items this launch: (B * n_tiles or n_tab) * (G / groups_per_cta)
  int r_lo, r_hi;    // packed query rows whose sel / scores this launch writes
  int32_t *sel;      // selection rows (see QGeo)
  float *scores;     // block-score rows (see QGeo), nb entries each
  int *status;
};
int index_groups_per_cta(int G, int top_k);
cudaError_t launch_index_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                                int num_sms, cudaStream_t st);

struct TopkArgs {
  int B, G, L, nb, top_k, blk;
  const float *scores;  // [B,G,L,nb]
  int32_t *sel;         // [B,G,L,top_k]
};
cudaError_t launch_topk_kernel(const TopkArgs &a, cudaStream_t st);

// Reverse index and attention over one query chunk: the packed rows
// [r0, r0 + Rc).  Per-entry arrays of the chunk (pos_of) are laid out
// [G][Rc][top_k].
struct RevIdxArgs {
  int G, nb, top_k, qpi;        // qpi: queries per 128-row tile (128 / (H/G))
  QGeo q;
  int r0, Rc;                   // query chunk
  const int32_t *sel;           // selection rows (see QGeo)
  int32_t *cnt;                 // [B*G*nb]      (zeroed by the launcher)
  int32_t *list_off;            // [B*G*nb + 1]
  int32_t *item_off;            // [B*G*nb + 1]
  int32_t *list;                // [G*Rc*top_k]: t * 32 + slot
  int32_t *pos_of;              // [G][Rc][top_k]: rank in its block's list, then list position
  // > 0: sort every list by query position (run-to-run stable order);
  // ceil(rows / 32) for the most rows one sequence has in a chunk
  int order_words;
  int *status;
};
cudaError_t launch_revidx(const RevIdxArgs &a, cudaStream_t st);
size_t revidx_order_smem(int order_words);   // shared memory of the ordering step

struct AttnArgs {
  int L, H, G, nb, top_k;      // L: key rows per sequence
  int blk;                     // block length: 128 or 64
  QGeo q;
  float scale, scale_log2;
  int max_items;               // upper bound on the chunk's work items
  const uint16_t *q_ptr;       // packed query rows [N,H,d]
  // Per-sequence K and V tensor maps in device memory ({K, V} of sequence b
  // at 2b, 2b+1; 4-D, batch extent 1), or null: the launch's own maps (4-D
  // over the whole batch).  Either way a map's row extent ends at the
  // sequence's last key, so rows past it load as zeros.
  const CUtensorMap *kv_maps;
  const int32_t *list;
  const int32_t *list_off;
  const int32_t *item_off;
  // Partials by reverse-index list position: entry pos owns rows pos*R + hh
  // (hh < R = H/G); a row's 16-byte granule c is stored at granule
  // c ^ (row & 7).
  uint16_t *part_o;            // [entries*R, d] bf16
  float *part_lse;             // [entries*R]
  int *status;
};
cudaError_t launch_prefill_attn(const CUtensorMap &tk, const CUtensorMap &tv, const AttnArgs &a,
                                int num_sms, cudaStream_t st);

struct CombineArgs {
  int H, G, top_k;
  QGeo q;
  int r0, Rc;                  // query chunk (packed rows)
  const int32_t *sel;          // selection rows (see QGeo)
  const int32_t *pos_of;       // [G][Rc][top_k]
  const uint16_t *part_o;      // see AttnArgs
  const float *part_lse;
  uint16_t *out;               // packed rows [N,H,d]
  float *lse;                  // packed rows [N,H] or null
};
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);

// Main-branch backward for the query chunk of packed rows [r0, r0 + Rc)
// (uniform batch, whole sequences: row b*L + t is position t of sequence b),
// over that chunk's reverse index.
struct BwdArgs {
  int B, L, H, G, nb, top_k;
  int blk;                     // block length: 128 or 64
  int r0, Rc;
  int last;                    // the last query chunk (writes dk, dv when chunked)
  float scale, scale_log2;
  const uint16_t *q;           // [B,L,H,d]
  const uint16_t *out, *dout;  // [B,L,H,d]: forward output and its gradient
  const float *lse;            // [B,L,H]: forward log-sum-exp (natural log)
  const int32_t *sel;          // [B,G,L,top_k]
  const int32_t *list, *list_off, *pos_of;   // reverse index of the chunk (see RevIdxArgs)
  float *delta;                // [B,L,H]: do . o
  // dq of (list position, head), scaled, bf16 [entries*R, d]; granule c
  // of partial row rho is stored at granule c ^ (rho & 7) (as AttnArgs)
  uint16_t *part_dq;
  uint16_t *dq;                // [B,L,H,d]
  uint16_t *dk, *dv;           // [B,L,G,d]
  // fp32 [B,L,G,d] dk/dv accumulators across query chunks (zeroed before the
  // first chunk), or null for a single chunk
  float *acc_dk, *acc_dv;
  int *unit_ctr;               // work counter (zeroed by the launcher)
  int *status;
};
// NSA-style branches (nsa_kernels.cu): query-outer exact attention over a
// contiguous visible key range per query row.
struct DenseAttnArgs {
  int B, L, H, G;              // queries q [B,L,H,d] (the tensor map's tensor)
  int n_qt;                    // query tiles per sequence: ceil(L / (128 / (H/G)))
  int mode;                    // 0: window over the tokens, 1: compressed tokens
  int window, blk;             // mode 0: s in [t-window+1, t]; mode 1: c <= (t+1)/blk - 1
  float scale, scale_log2;
  uint16_t *out;               // [B,L,H,d]
  float *lse;                  // [B,L,H] or null
  int *status;
};
cudaError_t launch_dense_attn(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                              const DenseAttnArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_nsa_compress(const uint16_t *k, const uint16_t *v, uint16_t *k_cmp,
                                uint16_t *v_cmp, int B, int L, int G, int blk, cudaStream_t st);
cudaError_t launch_nsa_gate(const float *gates, const uint16_t *o_cmp, const uint16_t *o_slc,
                            const uint16_t *o_win, uint16_t *out, long long rows, cudaStream_t st);

cudaError_t launch_bwd_delta(const BwdArgs &a, cudaStream_t st);   // D for all rows
cudaError_t launch_backward(const CUtensorMap &tk, const CUtensorMap &tv, const BwdArgs &a,
                            int num_sms, cudaStream_t st);      // one chunk: kernel + dq sums

struct DecodeArgs {
  int B, Lmax, H, G, d_idx, nb_max, top_k;
  int blk;                     // block length: 128 or 64 (nb_max = ceil(Lmax / blk))
  float scale, scale_log2;
  const uint16_t *q, *q_idx, *k_cache, *v_cache, *k_idx_cache;
  // FP8 index-key cache (when non-null, used instead of k_idx_cache):
  // E4M3 codes [B,Lmax,d_idx] and one fp32 scale per token [B,Lmax]
  const uint8_t *k_idx8;
  const float *k_idx_scale;
  // FP8 K/V caches (when non-null, used instead of k_cache / v_cache): E4M3
  // codes [B,Lmax,G,d] and one fp32 scale per (token, KV head) [B,Lmax,G]
  const uint8_t *k8, *v8;
  const float *k_scale, *v_scale;
  const int32_t *seq_lens;
  float *scores;               // [B,G,nb_max]
  int32_t *sel;                // [B,G,top_k]
  float *part_o;               // [B,H,top_k,d]
  float *part_lse;             // [B,H,top_k]
  int *tickets;                // [B,G]: merge tickets of the attention (zeroed by the top-k)
  uint16_t *out;               // [B,H,d]
  int *status;
};
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);

// Row-wise E4M3 quantization (one fp32 scale per row); cols % 8 == 0.
cudaError_t launch_quantize_e4m3_rows(const uint16_t *x, long long rows, int cols, uint8_t *codes,
                                      float *scale, cudaStream_t st);

// Sets the message msa_last_error() returns; returns `code`.
int report_error(int code, const char *msg);

// Unique id of the calling thread's current CUDA context (never reused by a
// later context, unlike a context handle or a device number); false when no
// context is current or the driver lacks the entry points.  Per-device state
// the library caches (device addresses of its own arrays, streams, events)
// is keyed on it, so a context rebuilt by cudaDeviceReset is not handed
// objects of the one it replaced.
bool current_context_id(unsigned long long *id);

}  // namespace msa
