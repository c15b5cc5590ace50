/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention library.
 *
 * The operation (cited by page title and section):
 *   Index Branch  -- "MiniMax M3 sparse attention" explainer
 *     (mlqm.cn/news/533796) §2.1: each GQA group has one index query
 *     q_idx[t,g]; all groups share one single-head index key k_idx[s]; the
 *     token score is q_idx . k_idx; "Block Max Pooling" turns token scores
 *     into block scores; top-k blocks are kept.
 *     "MiniMax Sparse Attention:百万上下文稀疏注意力" (researchpapers.dev),
 *     section "机制": only visible tokens (s <= t) are scored, the choice is
 *     per (query, group), the most recent local block is always kept.
 *   Main Branch   -- explainer §2.2: gather the selected K/V blocks and run
 *     ordinary softmax attention; every query head of a GQA group uses the
 *     group's selection.  researchpapers.dev section "2048 个 KV token":
 *     16 blocks x 128 tokens per query group.
 *   Decode        -- explainer §4.1: each new token scores the cache and
 *     attends only to its selected blocks.
 *   Backward      -- researchpapers.dev section "机制", training paragraph:
 *     the index branch is trained separately (KL loss) and its path into
 *     the main attention carries no gradient, so the main branch is
 *     differentiated with the selection held fixed.
 *
 * Definition implemented (readings where the pages are silent are marked R):
 *   S[b,g,t,j] = max_{s in block j, s <= t} sum_i q_idx[b,t,g,i]*k_idx[b,s,i]
 *                                          (R: raw dot product, no scale)
 *   sel[b,g,t] = {b_t} U top_(top_k-1){ S[b,g,t,j] : j < b_t },  b_t = t/block
 *                (R: top_k counts the local block; equal scores -> lower j;
 *                 if b_t+1 <= top_k every block 0..b_t is kept)
 *                stored sorted ascending, padded with -1.
 *   out[b,t,h] = softmax_s(scale * q[b,t,h].k[b,s,g]) . v[b,s,g]  over the
 *                tokens s <= t of the blocks in sel[b,g,t], g = h/(H/G).
 *                (R: scale = 1/sqrt(d) when params.scale == 0)
 *   dq, dk, dv = gradients of sum(dout * out) with respect to q, k, v, for
 *                a given sel (a constant).
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers, row-major, contiguous, 16-byte aligned.
 *     bf16 tensors are passed as raw 16-bit patterns (msa_bf16).
 *   - The caller owns every buffer, including the workspace `ws`
 *     (>= msa_workspace_bytes(p, op) bytes, 256-byte aligned).  The library
 *     allocates and frees nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and return once the work is queued.
 *   - The first 4 bytes of `ws` are a device status word.  Zero them once
 *     before the first call (e.g. allocate ws zeroed); the library only
 *     ever sets them to an error code, and msa_read_status() clears them.
 *   - Return value: MSA_OK or a negative MSA_ERR_* code; nothing is launched
 *     when a call returns an error.  msa_last_error() gives a message
 *     (thread-local).  Errors found on the device (a bounded wait that ran
 *     out, an out-of-range decode length) are recorded in a status word at
 *     the start of `ws`; msa_read_status() synchronises the stream and
 *     returns/clears it.
 *   - Supported: d == 128, d_idx in {64, 128}, block in {64, 128},
 *     1 <= top_k <= 32, H % G == 0 with H/G in {1,2,4,8,16}, B*L <= 2^26.
 *     Any L: the last block of a sequence may be partial (nb =
 *     ceil(L/block) blocks), in every operation.  The decode entry
 *     points also need G <= 8 (the cache scan scores all groups of a key in
 *     one 8-column tensor-core product).
 *     Other shapes give MSA_ERR_UNSUPPORTED.  B == 0 or L == 0 is a no-op.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t msa_bf16;   /* raw bfloat16 bits */
typedef void *msa_stream;    /* cudaStream_t */

typedef struct msa_params {
  int32_t B;       /* batch (prefill) / number of sequences (decode) */
  int32_t L;       /* sequence length (prefill) / cache capacity Lmax (decode) */
  int32_t H;       /* query heads */
  int32_t G;       /* GQA groups = KV heads = index queries per token */
  int32_t d;       /* head dim of q/k/v (128) */
  int32_t d_idx;   /* index dim of q_idx/k_idx (64 or 128) */
  int32_t block;   /* KV block length: 128 (the pages' size) or 64 */
  int32_t top_k;   /* blocks kept per (query, group), local block included */
  float scale;     /* softmax scale of the main branch; 0 -> 1/sqrt(d) */
  int32_t chunk;   /* query rows per chunk of the prefill attention and the
                      backward (rows of the packed batch, b*L + t), a
                      multiple of 128; 0 -> the longest chunk whose partials
                      fit the 16 GiB budget.  Smaller chunks need a smaller
                      workspace and re-read K/V more often. */
} msa_params;

enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = -1,    /* null/misaligned pointer, bad size */
  MSA_ERR_UNSUPPORTED = -2,    /* shape outside the supported set */
  MSA_ERR_WORKSPACE = -3,      /* ws too small or misaligned */
  MSA_ERR_CUDA = -4,           /* a CUDA runtime/driver call failed */
  MSA_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait ran out */
  MSA_ERR_DEVICE_INPUT = -6    /* device-side check failed (decode length) */
};

enum {
  MSA_OP_INDEX_SELECT = 0,
  MSA_OP_PREFILL_ATTN = 1,
  MSA_OP_DECODE = 2,
  MSA_OP_FORWARD = 3,
  MSA_OP_BACKWARD = 4,
  MSA_OP_FORWARD_VARLEN = 5,
  MSA_OP_NSA_BRANCH = 6,     /* msa_nsa_window_attn, msa_nsa_compressed_attn */
  MSA_OP_NSA_FORWARD = 7     /* msa_nsa_forward */
};

/* Index Branch (explainer §2.1; researchpapers.dev "机制").
 *   q_idx  [B,L,G,d_idx] bf16, k_idx [B,L,d_idx] bf16            (in)
 *   sel    [B,G,L,top_k] int32                                    (out)
 *   block_scores [B,G,L,nb] fp32, nb = ceil(L/block), or NULL       (out)
 *     When given, entry (t, j) holds S[b,g,t,j] for j < t/block and -inf
 *     for j >= t/block (the local block is forced, never scored), and sel
 *     is computed from these stored scores by the top-k kernel.  When NULL
 *     the top-k runs inside the index kernel's epilogue and the L x nb
 *     score matrix never reaches memory; both routes give the same sel.
 */
int msa_index_select(const msa_params *p, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                     int32_t *sel, float *block_scores, void *ws, size_t ws_bytes,
                     msa_stream stream);

/* Main Branch, prefill (explainer §2.2; researchpapers.dev "机制").
 *   q [B,L,H,d], k [B,L,G,d], v [B,L,G,d] bf16                      (in)
 *   sel [B,G,L,top_k] int32: any selection in the layout above: valid
 *     ids first (any order, each < nb, each block at most once, the
 *     query's own block included for a causal result), -1 padding.   (in)
 *   out [B,L,H,d] bf16                                              (out)
 *   lse [B,L,H] fp32 natural-log softmax normaliser, or NULL         (out)
 * Blocks are processed key-block-outer: queries that chose the same block
 * are gathered into 128-row tiles (reverse index), per-block partial
 * results are merged at the end.
 */
int msa_sparse_attn_prefill(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k,
                            const msa_bf16 *v, const int32_t *sel, msa_bf16 *out,
                            float *lse, void *ws, size_t ws_bytes, msa_stream stream);

/* Decode step (explainer §4.1).  p->B = sequences, p->L = cache capacity.
 *   q [B,H,d], q_idx [B,G,d_idx] bf16: the new token's queries       (in)
 *   k_cache, v_cache [B,Lmax,G,d], k_idx_cache [B,Lmax,d_idx] bf16   (in)
 *   seq_lens [B] int32 DEVICE array: cached tokens per sequence, the new
 *     token's k/v/k_idx already appended, so the query sits at position
 *     seq_lens[b]-1.  Values outside [1, Lmax] set MSA_ERR_DEVICE_INPUT in
 *     the status word and that sequence's output is zero.              (in)
 *   out [B,H,d] bf16                                                (out)
 *   sel [B,G,top_k] int32 or NULL: the blocks used                  (out)
 */
int msa_sparse_attn_decode(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                           const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                           const msa_bf16 *k_idx_cache, const int32_t *seq_lens,
                           msa_bf16 *out, int32_t *sel, void *ws, size_t ws_bytes,
                           msa_stream stream);

/* Decode step with the index-key cache stored in FP8 (the essay's low-
 * precision cache direction): the stored index key of token s is
 * k_idx_scale[s] * E4M3(k_idx8[s]), E4M3 being the OCP 8-bit floating-point
 * format (4 exponent bits, bias 7, 3 mantissa bits).  The scan, most of a
 * decode step's bytes, reads half as much.  Everything else is
 * msa_sparse_attn_decode.
 *   k_idx8 [B,Lmax,d_idx] uint8 E4M3 codes, 16-byte aligned           (in)
 *   k_idx_scale [B,Lmax] fp32, one scale per token                      (in)
 * Scores are accumulated in fp32 from f16 products: q_idx must lie within
 * the f16 range (|x| < 65504), where its bf16 values convert exactly.
 * msa_quantize_e4m3_rows produces codes and scales from bf16 rows. */
int msa_sparse_attn_decode_fp8idx(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                                  const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                                  const uint8_t *k_idx8, const float *k_idx_scale,
                                  const int32_t *seq_lens, msa_bf16 *out, int32_t *sel, void *ws,
                                  size_t ws_bytes, msa_stream stream);

/* Decode step with every cache in FP8: the index keys as in
 * msa_sparse_attn_decode_fp8idx, and the keys and values as E4M3 codes
 * with one fp32 scale per (token, KV head): the stored key of token s,
 * head g is k_scale[s,g] * E4M3(k8[s,g,:]), likewise for values.
 *   k8, v8 [B,Lmax,G,d] uint8 E4M3 codes, 16-byte aligned             (in)
 *   k_scale, v_scale [B,Lmax,G] fp32                                    (in)
 *   k_idx8 [B,Lmax,d_idx] uint8, k_idx_scale [B,Lmax] fp32              (in)
 * The main branch's scores run in f16 (q must lie within the f16 range);
 * each value's scale is folded into its softmax weight before the weights
 * are rounded to bf16 for the P V product. */
int msa_sparse_attn_decode_fp8(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                               const uint8_t *k8, const float *k_scale, const uint8_t *v8,
                               const float *v_scale, const uint8_t *k_idx8,
                               const float *k_idx_scale, const int32_t *seq_lens, msa_bf16 *out,
                               int32_t *sel, void *ws, size_t ws_bytes, msa_stream stream);

/* Quantize `rows` bf16 rows of `cols` values (cols a multiple of 16) to
 * E4M3 codes with one fp32 scale per row: scale = max|x| / 448 (1 for an
 * all-zero row), code = E4M3 round-to-nearest-even of x / scale, saturated
 * to +-448.  x [rows, cols] bf16 (in); codes [rows, cols] uint8, scale
 * [rows] fp32 (out).  Device pointers, 16-byte aligned. */
int msa_quantize_e4m3_rows(const msa_bf16 *x, long long rows, int cols, uint8_t *codes,
                           float *scale, msa_stream stream);

/* Decode step without a workspace argument, for callers that cannot
 * allocate device memory where they run a decode step (engines that plan all
 * device buffers at start-up and forbid allocation afterwards, plugin hosts
 * that pass a library only the call's tensors).  The pages have no
 * counterpart; this is a deployment convenience.
 *   Arguments and results are those of msa_sparse_attn_decode, minus ws.
 *   Scratch: a 16 MiB array in device memory owned by the library (every GPU
 *     that loads the library keeps it reserved until the process exits).
 *     Problems needing more scratch than that (msa_workspace_bytes(p,
 *     MSA_OP_DECODE) > 16 MiB, e.g. 32 sequences at 1M tokens) return
 *     MSA_ERR_WORKSPACE without launching anything.
 *   The first call on each device looks the array's device address up with
 *     cudaGetSymbolAddress; make that first call before any stream capture.
 *     The address is cached with the id of the context it belongs to and is
 *     looked up again in a new context (after cudaDeviceReset, or under
 *     another driver-API context on the device).
 *   All calls on a device share the array and it keeps the last call's
 *     contents: calls whose GPU work overlaps (other streams) race, so order
 *     them.  Device-side input errors are not reported by this variant (its
 *     status word is cleared on every call); an out-of-range length still
 *     yields a zero output for that sequence.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int msa_sparse_attn_decode_noalloc(const msa_params *p, const msa_bf16 *q, const msa_bf16 *q_idx,
                                   const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                                   const msa_bf16 *k_idx_cache, const int32_t *seq_lens,
                                   msa_bf16 *out, int32_t *sel, msa_stream stream);

/* Whole prefill: msa_index_select (fused top-k) then msa_sparse_attn_prefill.
 *   sel may be NULL (kept in ws); lse may be NULL.                      */
int msa_forward(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k, const msa_bf16 *v,
                const msa_bf16 *q_idx, const msa_bf16 *k_idx, msa_bf16 *out, int32_t *sel,
                float *lse, void *ws, size_t ws_bytes, msa_stream stream);

/* Prefill of n new tokens per sequence, at positions [t0, t0 + n), against
 * a cache that already holds every key up to t0 + n: the serving form of
 * the prefill (a prompt processed in chunks, or continued after a cached
 * prefix; the explainer's serving discussion, §4.1).  Each new query attends
 * exactly as in msa_forward over a sequence of length t0 + n, so the
 * results equal rows [t0, t0 + n) of that call.
 *   p->L = cache capacity Lmax; any t0, n >= 0 with t0 + n <= Lmax
 *   q [B,n,H,d], q_idx [B,n,G,d_idx] bf16: the new tokens' queries     (in)
 *   k_cache, v_cache [B,Lmax,G,d], k_idx_cache [B,Lmax,d_idx] bf16, the
 *     new tokens' rows already written; rows >= t0 + n are not read     (in)
 *   out [B,n,H,d] bf16; sel [B,G,n,top_k] int32 or NULL; lse [B,n,H]
 *     fp32 or NULL                                                   (out)
 *   ws >= msa_workspace_bytes(p, MSA_OP_FORWARD)
 * Every sequence of the batch has the same t0 and n. */
int msa_forward_cached(const msa_params *p, int t0, int n, const msa_bf16 *q,
                       const msa_bf16 *q_idx, const msa_bf16 *k_cache, const msa_bf16 *v_cache,
                       const msa_bf16 *k_idx_cache, msa_bf16 *out, int32_t *sel, float *lse,
                       void *ws, size_t ws_bytes, msa_stream stream);

/* msa_forward_cached for a batch whose sequences continue at different
 * positions with different numbers of new tokens (a ragged serving batch).
 * The new tokens' query rows are packed: sequence b owns rows
 * [row0_b, row0_b + n[b]) with row0_b = n[0] + ... + n[b-1].
 *   t0[B], n[B]: HOST int32 arrays; any t0[b], n[b] >= 0 with
 *     t0[b] + n[b] <= Lmax (n[b] may be 0)
 *   q [sum n, H, d], q_idx [sum n, G, d_idx] bf16 (packed)              (in)
 *   k_cache, v_cache [B,Lmax,G,d], k_idx_cache [B,Lmax,d_idx]            (in)
 *   out [sum n, H, d] bf16 (packed); lse [sum n, H] fp32 or NULL        (out)
 *   ws >= msa_workspace_bytes(p, MSA_OP_FORWARD_VARLEN)
 * The whole batch runs in one launch per kernel (per query chunk of
 * packed rows): the call builds, on the host, each sequence's K/V tensor
 * maps (row extent t0[b] + n[b], so keys past a sequence's end are never
 * read), the per-sequence query geometry and the index branch's list of
 * (sequence, 128-query tile) work items, longest first, and uploads them
 * into ws with one cudaMemcpyAsync (from pageable memory: the call returns
 * once they are staged).  Every row equals msa_forward_cached's row for its
 * sequence. */
int msa_forward_cached_varlen(const msa_params *p, const int32_t *t0, const int32_t *n,
                              const msa_bf16 *q, const msa_bf16 *q_idx, const msa_bf16 *k_cache,
                              const msa_bf16 *v_cache, const msa_bf16 *k_idx_cache,
                              msa_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                              msa_stream stream);

/* Device buffers that msa_forward_host stages its transfers in: the device
 * counterparts of msa_forward's tensors (caller-owned, 16-byte aligned).
 * lse may be NULL when no lse is requested. */
typedef struct msa_staging {
  msa_bf16 *q, *k, *v, *q_idx, *k_idx;   /* inputs, device copies   */
  msa_bf16 *out;                          /* [B,L,H,d] device output */
  float *lse;                             /* [B,L,H] or NULL         */
} msa_staging;

/* msa_forward with inputs and outputs in HOST memory, transfers overlapped
 * with the computation.  There is no counterpart in the pages; this is the
 * end-to-end path of a caller whose tensors live in host memory.
 *   q_h, k_h, v_h, q_idx_h, k_idx_h  host inputs, layouts of msa_forward (in)
 *   out_h [B,L,H,d] bf16, lse_h [B,L,H] fp32 or NULL: host outputs      (out)
 *   dev       device staging buffers (dev->lse needed iff lse_h)
 *   ws        as msa_forward (msa_workspace_bytes(p, MSA_OP_FORWARD))
 *   stream    compute stream;  copy_stream  the transfers (may equal stream,
 *             which serialises them with the computation)
 * Order of work, per query chunk [t0, t0+Lc) (msa_prefill_chunk_len): the
 * chunk's rows of k_idx and q_idx go up on copy_stream, then its rows of k,
 * v and q; on `stream` the index branch runs for the chunk's query tiles as
 * soon as its index rows are up, then the main branch for its queries; the
 * chunk's output rows (and lse) come down on a download stream of the
 * library as soon as the chunk is merged.  A chunk needs only rows < t0+Lc,
 * so transfers and computation of neighbouring chunks overlap.  When the
 * call returns everything is enqueued, and work later enqueued on `stream`
 * runs after the last download, so synchronising `stream` makes out_h
 * valid.  Host buffers must be pinned (page-locked) for the copies to
 * overlap; pageable buffers still give correct results.  Uses four CUDA
 * events and one stream per device, created on the first call on that
 * device and reused; calls from several host threads are serialised while
 * they enqueue. */
int msa_forward_host(const msa_params *p, const msa_bf16 *q_h, const msa_bf16 *k_h,
                     const msa_bf16 *v_h, const msa_bf16 *q_idx_h, const msa_bf16 *k_idx_h,
                     msa_bf16 *out_h, float *lse_h, const msa_staging *dev, void *ws,
                     size_t ws_bytes, msa_stream stream, msa_stream copy_stream);

/* Main Branch, backward pass (researchpapers.dev "机制", training
 * paragraph: the index path is cut from the main attention's gradient, so
 * the selection is a constant and only q, k and v receive gradients).
 *   q [B,L,H,d], k [B,L,G,d], v [B,L,G,d] bf16: forward inputs        (in)
 *   out [B,L,H,d] bf16, lse [B,L,H] fp32: msa_sparse_attn_prefill's
 *     outputs for the same inputs and selection                       (in)
 *   dout [B,L,H,d] bf16: gradient of the loss with respect to out     (in)
 *   sel [B,G,L,top_k] int32: the forward's selection                  (in)
 *   dq [B,L,H,d], dk [B,L,G,d], dv [B,L,G,d] bf16                    (out)
 * For each (t, h) with probabilities P over its attended tokens s:
 * dZ_s = P_s (do . v_s - do . o), dq = scale sum_s dZ_s k_s, and every
 * attended token gets dk_s += scale dZ_s q, dv_s += P_s do; tokens no query
 * attends to get zero.  dq, dk and dv are bit-identical from run to run:
 * dq sums a row's slots in slot order, and dk and dv sum a key block's
 * queries in query order (the reverse index's lists are sorted).
 * Any L and either block length: the block that holds a sequence's last
 * key is partial, and a 64-token block fills half of the kernel's 128-key
 * tile (the other half is masked out).  Queries are processed in the
 * prefill's chunks of packed rows (msa_prefill_chunk_len; p->chunk
 * overrides it), at most 2^19 rows each, each with its
 * own reverse index and one bf16 dq partial row per (query, head, slot) of
 * the chunk (at most about 16 GiB).
 * With more than one chunk, dk and dv are summed across chunks in fp32
 * accumulators (2 * B*L*G*d*4 bytes of workspace) and rounded to bf16 once.
 * ws >= msa_workspace_bytes(p, MSA_OP_BACKWARD). */
int msa_sparse_attn_backward(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k,
                             const msa_bf16 *v, const msa_bf16 *out, const float *lse,
                             const msa_bf16 *dout, const int32_t *sel, msa_bf16 *dq,
                             msa_bf16 *dk, msa_bf16 *dv, void *ws, size_t ws_bytes,
                             msa_stream stream);

/* ---- NSA-style variant --------------------------------------------------
 * "MiniMax M3 sparse attention" explainer (mlqm.cn/news/533796), §3.1:
 * DeepSeek NSA runs three parallel branches -- compression, selection and a
 * sliding window -- mixed by a learned gate; MSA keeps the selection alone.
 * These entry points add the other two branches beside MSA's selection.
 * The page gives them no formulas; the readings implemented:
 *   window       query t attends its `window` most recent tokens, s in
 *                [t-window+1, t] (exact softmax attention, scale as p);
 *   compression  compressed token c is the mean of block c's keys (values),
 *                block = p->block; query t attends the compressed tokens of
 *                the blocks whose every token lies at or before t, i.e.
 *                c <= (t+1)/block - 1; a query with none gets a zero output
 *                (lse -inf);
 *   gate         three gates per (query, head) from the caller (the learned
 *                gate needs trained weights); out = g_cmp o_cmp + g_slc o_slc
 *                + g_win o_win, accumulated in fp32.
 * Layouts as above; k_cmp, v_cmp [B,nb,G,d] bf16 with nb = ceil(L/block);
 * gates [B,L,H,3] fp32 in the order (cmp, slc, win).  Same shape support
 * as the prefill.  Every branch kernel is query-outer: a 128-row tile of
 * 128/(H/G) consecutive queries x H/G heads sweeps the key tiles its rows
 * see once, accumulating P V in TMEM (rescaled in place when a row's
 * maximum grows). */

/* Compressed keys and values: k_cmp[b,c,g] = mean of k[b,s,g] over the
 * tokens s of block c (a partial last block averages the tokens it has),
 * fp32 sums rounded to bf16; the same for v.  No workspace. */
int msa_nsa_compress_kv(const msa_params *p, const msa_bf16 *k, const msa_bf16 *v,
                        msa_bf16 *k_cmp, msa_bf16 *v_cmp, msa_stream stream);

/* Sliding-window branch: out [B,L,H,d] bf16 and (nullable) lse [B,L,H]
 * fp32 of each query over its window >= 1 most recent tokens.
 * ws >= msa_workspace_bytes(p, MSA_OP_NSA_BRANCH) (the status word). */
int msa_nsa_window_attn(const msa_params *p, int32_t window, const msa_bf16 *q,
                        const msa_bf16 *k, const msa_bf16 *v, msa_bf16 *out, float *lse,
                        void *ws, size_t ws_bytes, msa_stream stream);

/* Compression branch: out, lse of each query over the compressed tokens
 * of its completed blocks (msa_nsa_compress_kv's output).
 * ws >= msa_workspace_bytes(p, MSA_OP_NSA_BRANCH). */
int msa_nsa_compressed_attn(const msa_params *p, const msa_bf16 *q, const msa_bf16 *k_cmp,
                            const msa_bf16 *v_cmp, msa_bf16 *out, float *lse, void *ws,
                            size_t ws_bytes, msa_stream stream);

/* out = g_cmp o_cmp + g_slc o_slc + g_win o_win per (b, t, h); out may be
 * one of the three inputs.  No workspace. */
int msa_nsa_gate(const msa_params *p, const float *gates, const msa_bf16 *o_cmp,
                 const msa_bf16 *o_slc, const msa_bf16 *o_win, msa_bf16 *out,
                 msa_stream stream);

/* The whole NSA-style prefill: MSA's index branch and selection branch
 * (as msa_forward), the compression and window branches, and the gate.
 * sel [B,G,L,top_k] is nullable.
 * ws >= msa_workspace_bytes(p, MSA_OP_NSA_FORWARD): msa_forward's, plus
 * k_cmp, v_cmp and two branch outputs (the selection branch's output is
 * written to out and gated in place). */
int msa_nsa_forward(const msa_params *p, int32_t window, const msa_bf16 *q, const msa_bf16 *k,
                    const msa_bf16 *v, const msa_bf16 *q_idx, const msa_bf16 *k_idx,
                    const float *gates, msa_bf16 *out, int32_t *sel, void *ws, size_t ws_bytes,
                    msa_stream stream);

/* Workspace bytes op (MSA_OP_*) needs for these params; 0 when p is invalid
 * (see msa_last_error). */
size_t msa_workspace_bytes(const msa_params *p, int op);

/* Query-chunk length the prefill attention uses for these params: the
 * packed query rows (b*L + t) are processed in chunks of this many rows so
 * that per-block partial results stay within a fixed workspace budget
 * (about 16 GiB).  Each chunk costs 5 kernel launches.  0 when p is
 * invalid. */
int msa_prefill_chunk_len(const msa_params *p);

/* Synchronise `stream`, return the device status recorded in ws (MSA_OK or
 * MSA_ERR_DEVICE_*), and reset it to MSA_OK. */
int msa_read_status(void *ws, msa_stream stream);

/* Message of the last error on this host thread ("" if none). */
const char *msa_last_error(void);

/* Library version string. */
const char *msa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
