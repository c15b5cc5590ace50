// Internal launch interface between the C-ABI layer (msa_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace msa {

// Query-side tensors (q, q_idx, sel, scores, out, lse) hold Lq rows per
// sequence, row 0 being position tq0; key-side tensors (k, v, k_idx) hold
// L rows per sequence from position 0.  A whole-sequence call has Lq = L,
// tq0 = 0.
struct IndexArgs {
  int B, L, G, nb, top_k, d_idx;
  int Lq, tq0;
  int write_scores;  // 1: store block scores, 0: fused top-k -> sel
  int i_hi;          // query tiles [i_hi - n_items / (B * G/groups_per_cta), i_hi)
  int n_items;       // B * (query tiles) * (G / groups_per_cta)
  int32_t *sel;      // [B,G,L,top_k]
  float *scores;     // [B,G,L,nb]
  int *status;
};
int index_groups_per_cta(int G, int top_k);
cudaError_t launch_index_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const IndexArgs &a,
                                int num_sms, cudaStream_t st);

struct TopkArgs {
  int B, G, L, nb, top_k;
  const float *scores;  // [B,G,L,nb]
  int32_t *sel;         // [B,G,L,top_k]
};
cudaError_t launch_topk_kernel(const TopkArgs &a, cudaStream_t st);

struct RevIdxArgs {
  int B, G, L, nb, top_k, qpi;  // qpi: queries per 128-row tile (128 / (H/G))
  int Lq, tq0;                  // query-side geometry (see IndexArgs)
  int t0, Lc;                   // query chunk [t0, t0 + Lc)
  const int32_t *sel;           // [B,G,L,top_k]
  int32_t *cnt;                 // [B*G*nb]      (zeroed by the caller)
  int32_t *list_off;            // [B*G*nb + 1]
  int32_t *item_off;            // [B*G*nb + 1]
  int32_t *list;                // [B*G*Lc*top_k]
  int32_t *pos_of;              // [B,G,Lc,top_k]: rank in its block's list, then list position
  int *status;
};
cudaError_t launch_revidx(const RevIdxArgs &a, cudaStream_t st);

struct AttnArgs {
  int B, L, H, G, nb, top_k;
  int Lq, tq0;                 // query-side geometry (see IndexArgs)
  float scale, scale_log2;
  int t0, Lc;
  int max_items;               // upper bound on the chunk's work items
  const uint16_t *q;           // [B,L,H,d]
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
  int B, L, H, G, top_k;
  int Lq, tq0;                 // query-side geometry (see IndexArgs)
  int t0, Lc;
  const int32_t *sel;          // [B,G,L,top_k]
  const int32_t *pos_of;       // [B,G,Lc,top_k]
  const uint16_t *part_o;      // see AttnArgs
  const float *part_lse;
  uint16_t *out;               // [B,L,H,d]
  float *lse;                  // [B,L,H] or null
};
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);

// Main-branch backward for the query chunk [t0, t0 + Lc), over that chunk's
// reverse index.
struct BwdArgs {
  int B, L, H, G, nb, top_k;
  int t0, Lc;
  int last;                    // the last query chunk (writes dk, dv when chunked)
  float scale, scale_log2;
  const uint16_t *q;           // [B,L,H,d]
  const uint16_t *out, *dout;  // [B,L,H,d]: forward output and its gradient
  const float *lse;            // [B,L,H]: forward log-sum-exp (natural log)
  const int32_t *sel;          // [B,G,L,top_k]
  const int32_t *list, *list_off, *pos_of;   // reverse index (see RevIdxArgs)
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
cudaError_t launch_bwd_delta(const BwdArgs &a, cudaStream_t st);   // D for all rows
cudaError_t launch_backward(const CUtensorMap &tk, const CUtensorMap &tv, const BwdArgs &a,
                            int num_sms, cudaStream_t st);      // one chunk: kernel + dq sums

struct DecodeArgs {
  int B, Lmax, H, G, d_idx, nb_max, top_k;
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
