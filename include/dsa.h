/*
 * dsa.h -- C ABI of libdsa: the decode step of a DeepSeek-Sparse-Attention
 * (DSA) layer and of a sliding-window (SWA) layer, for NVIDIA B200 (sm_100a).
 *
 * What is computed (sources: the explainer page "Naive-N0.5-Flash: no
 * full-attention layers, and a runtime built by AI"):
 *   - property table: 16 index heads x 128, one shared index-key head in
 *     fp8_e4m3; top 2,048 keys per DSA query; SWA window 128; 64 query heads,
 *     qk head dim 192, v head dim 128; 4 KV heads on DSA layers (GQA4), 8 on
 *     SWA layers (GQA8); native context 1,048,576.
 *   - "Inside a DSA layer: the lightning indexer": every visible key gets one
 *     score, relu(q_h . k) per index head combined by a per-head weight; the
 *     main heads attend only to the top-scoring 2,048 keys; the SWA heads carry
 *     a sink column in the softmax.
 *   - "What 'no full-attention layers' means": SWA masks keys with
 *     query_offset - key_offset >= window; DSA takes the first top_k entries
 *     of an argsort of the scores (ties toward the lower position, "How much
 *     of this did AI actually build?").
 *
 * Conventions shared by every call
 *   - All pointers named as device pointers must point to device (or managed)
 *     memory of the current CUDA device.  The caller owns every buffer; the
 *     library allocates nothing.  Scratch memory is the caller's workspace
 *     (`ws`, `ws_bytes`); `dsa_workspace_size` gives the size each call needs.
 *     A workspace must be zero when first used (`dsa_workspace_init`).  The
 *     parts that must start at zero (the selection's cross-CTA scratch and
 *     barrier words) are zeroed again by each call before it finishes; the
 *     status word keeps device errors until `dsa_check_device_status` reads
 *     it; scores, selections and attention partials are simply overwritten.
 *     After a device error (a wait that ran out) re-initialise the workspace.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream).  Host-side argument checks return before anything is
 *     enqueued.  Device-side checks (positions out of range, a bounded wait
 *     that ran out) set a status word in the workspace instead of faulting;
 *     read it with `dsa_check_device_status`.
 *   - Return value: DSA_OK or a DSA_ERR_* code; `dsa_last_error()` gives a
 *     thread-local message for the last failing call on this thread.  No C++
 *     exception crosses this boundary.
 *   - Calls that use the same workspace must not overlap in time.
 *   - Positions are 0-based int32.  Query (b, t) sits at position
 *     q_pos[b*T + t] and sees keys 0..q_pos[b*T + t] of its sequence.
 *
 * Tensor layouts (row-major, innermost last; "rows" are KV-cache rows, see
 * dsa_kv_t):
 *   q8       uint8 (e4m3 codes) [B][T][16][128]   index queries
 *   q_scale  float [B][T][16]                      index-query scales (> 0)
 *   w        float [B][T][16]                      index-head weights
 *   Q        bf16  [B][T][64][192]                 backbone queries
 *   O        bf16  [B][T][64][128]                 attention output
 *   lse      float [B][T][64]                      optional: natural-log
 *            sum-exp of the logits including the sink, log(sum_i e^{s_i} + e^{sink})
 *   scores   float [B][T][scores_stride]           indexer output
 *   idx      int32 [B][T][top_k]                   selected positions, -1 padded
 *   count    int32 [B][T]                          number of valid entries of idx
 *   sink     float [64]                            optional per-head sink logits
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define DSA_OK                      0
#define DSA_ERR_INVALID_ARG         1  /* null pointer, negative size, bad stride ... */
#define DSA_ERR_UNSUPPORTED_SHAPE   2  /* head dims, T, top_k, page size outside what is built */
#define DSA_ERR_WORKSPACE_TOO_SMALL 3
#define DSA_ERR_CUDA                4  /* a CUDA runtime call failed; see dsa_last_error() */
#define DSA_ERR_DEVICE_TIMEOUT      5  /* a bounded device-side wait ran out */
#define DSA_ERR_DEVICE_BAD_INDEX    6  /* a device-side position/page index was out of range */

/* Compile-time model dimensions (property table of the explainer page). */
#define DSA_INDEX_HEADS 16
#define DSA_INDEX_DIM   128
#define DSA_Q_HEADS     64
#define DSA_QK_DIM      192
#define DSA_V_DIM       128
#define DSA_MAX_TOPK    2048   /* largest top_k the selection kernel supports */
#define DSA_MAX_T       16     /* query tokens per sequence per decode call */

/* Operation ids for dsa_workspace_size. */
#define DSA_OP_INDEXER     0
#define DSA_OP_TOPK        1
#define DSA_OP_SPARSE_ATTN 2
#define DSA_OP_SWA_ATTN    3
#define DSA_OP_LAYER       4
#define DSA_OP_PREFILL     5   /* B = 1, T = NQ query tokens of dsa_prefill */
#define DSA_OP_PRODUCE     6   /* dsa_index_produce (the status word only) */
#define DSA_OP_KL          7   /* dsa_indexer_kl */

/*
 * KV-cache description.  One "row" holds one position of one sequence:
 *   k            bf16  [rows][num_kv_heads][192]   backbone keys (post-RoPE)
 *   v            bf16  [rows][num_kv_heads][128]   backbone values
 *   index_k      uint8 [rows][128]                 e4m3 index keys
 *   index_k_scale float [rows]                     per-row index-key scales (> 0)
 * The row of position `pos` of sequence `b` is
 *   contiguous (block_table == NULL): b * seq_stride + pos, pos < seq_stride
 *   paged:  block_table[b * max_pages + pos / page_size] * page_size + pos % page_size,
 *           pos / page_size < max_pages; page ids < num_rows / page_size.
 * `num_rows` is the number of rows the buffers hold (bounds every access).
 * Unused members may be NULL (e.g. index_k for the attention calls, k / v
 * for the indexer).  All device pointers must be 16-byte aligned.  The
 * indexer calls with B > 1 on a contiguous cache need seq_stride % 16 == 0.
 */
typedef struct dsa_kv {
    const void    *k;
    const void    *v;
    const void    *index_k;
    const float   *index_k_scale;
    int32_t        num_kv_heads;   /* G: 4 on DSA layers, 8 on SWA layers (any divisor of 64 up to 16 heads per group) */
    int32_t        page_size;      /* paged only: rows per page, a multiple of 16 dividing 128 or a multiple of 128 */
    int64_t        seq_stride;     /* contiguous only: rows reserved per sequence */
    int64_t        num_rows;       /* rows held by the buffers */
    const int32_t *block_table;    /* device int32 [B][max_pages], or NULL for contiguous */
    int32_t        max_pages;      /* row stride of block_table */
    int32_t        reserved;
} dsa_kv_t;

/* Thread-local message describing the last error returned on this thread. */
const char *dsa_last_error(void);

/* Writes the compiled dims {16, 128, 64, 192, 128, DSA_MAX_TOPK, DSA_MAX_T}
 * to dims[0..n) (n <= 7) and returns DSA_OK. */
int dsa_get_dims(int32_t *dims, int n);

/* Workspace bytes that operation `op` (DSA_OP_*) needs for a call with B
 * sequences, T query tokens each, contexts of at most Lmax positions and the
 * given top_k (window for DSA_OP_SWA_ATTN).  Writes *bytes and returns DSA_OK,
 * or an error for unsupported arguments. */
int dsa_workspace_size(int op, int B, int T, int64_t Lmax, int top_k, size_t *bytes);

/* Zeroes a workspace (cudaMemsetAsync on `stream`). */
int dsa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Synchronises `stream`, then reads the device status word held in the
 * workspace and clears its error bits.  *status receives DSA_OK,
 * DSA_ERR_DEVICE_TIMEOUT or DSA_ERR_DEVICE_BAD_INDEX; *flags (if not NULL)
 * receives the whole word: bit (1 << code) for each kind of error seen, and
 * DSA_STATUS_NEEDS_INIT when a cross-CTA wait ran out.
 * After a timeout the workspace must be re-initialised with
 * dsa_workspace_init: DSA_STATUS_NEEDS_INIT stays set until then (reading the
 * status does not clear it), and until then the calls that use the
 * workspace's cross-CTA scratch (dsa_topk_select with more than one CTA per
 * row, dsa_layer_decode, dsa_prefill) compute nothing and report
 * DSA_ERR_DEVICE_TIMEOUT again, instead of running on a half-updated
 * scratch. */
#define DSA_STATUS_NEEDS_INIT 0x80000000u
int dsa_check_device_status(void *ws, void *stream, int *status, uint32_t *flags);

/* Synchronises `stream`, then reads two counters that the workspace header
 * keeps since its last dsa_workspace_init: how many dsa_layer_decode calls
 * (and dsa_layer_chain DSA steps) ran the one-barrier kernel for up to four
 * long query rows on its fast path (*fast: the key stream's sampled threshold
 * left between top_k and 16,384 candidates in every row, none lost) and on its
 * general path (*general: a full selection over the stored scores).  Both
 * give the same outputs; the counters say what the call cost.  Other paths
 * count in neither.  Counters wrap at 2^32.  No page counterpart: an
 * interface of this library. */
int dsa_layer_path_counts(void *ws, void *stream, uint32_t *fast, uint32_t *general);

/* Failure injection, for tests of the device-side failure path (no page
 * counterpart; an interface of this library).  While DSA_INJECT_BARRIER_TIMEOUT
 * is set (process-wide, for launches made from any host thread), every launch
 * of a kernel whose CTAs wait on one another (dsa_topk_select with more than
 * one CTA per row, the fused dsa_layer_decode) makes its first cross-CTA
 * barrier wait for one arrival more than will ever come, and bounds that wait
 * by wait_limit_ns (1e3 .. 1e9) instead of the normal 2 s: the wait runs out,
 * the kernel records DSA_ERR_DEVICE_TIMEOUT (and DSA_STATUS_NEEDS_INIT) in the
 * workspace and returns, and the GPU stays usable.  Nothing faults or hangs.
 * DSA_INJECT_NONE (wait_limit_ns ignored) restores normal operation.
 * Returns DSA_ERR_INVALID_ARG for an unknown kind or limit. */
#define DSA_INJECT_NONE            0
#define DSA_INJECT_BARRIER_TIMEOUT 1
int dsa_debug_inject(int kind, int64_t wait_limit_ns);

/* Phase trace of the one-barrier layer-step kernel (dsa_layer_decode and the
 * DSA steps of dsa_layer_chain for up to four long query rows), for
 * profiling; no page counterpart.  While a buffer is set (process-wide; NULL
 * or words == 0 switches it off), every launch of that kernel made with a
 * grid of at most words / DSA_TRACE_MARKS CTAs writes, per CTA c, the GPU's
 * nanosecond clock (%globaltimer) into buf[c * DSA_TRACE_MARKS + i]:
 *   i = 0 entry, 1 the sampled thresholds seen, 2 the key stream done (the
 *   CTA's tiles scored), 3 past the grid barrier, 4 the
 *   selection done, 5 the attention units done, 6 exit, 7 the CTA's sample
 *   handed in, 8 the candidate list in shared memory, 9 the k-th key found
 *   (radix select done), 10 the first key tile requested, 11 its MMA issued,
 *   12 its scores in the epilogue; 13 and 14 the SM's cycle counter
 *   (clock64) at entry and at exit, for the clock rate; 15 the CTA's
 *   candidates captured (after its tiles, from their stored scores).
 * Marks a CTA does not reach (a CTA with no selection or attention work, the
 * general path) are written as 0.  `buf` is device memory of the caller's,
 * `words` its length in uint64 words; a launch with a grid too large for it
 * writes nothing.  The buffer must outlive the launches made while it is
 * set.  Returns DSA_ERR_INVALID_ARG for words < 0 or a NULL buf with words > 0. */
#define DSA_TRACE_MARKS 16
int dsa_trace_phases(uint64_t *buf, int64_t words);

/*
 * dsa_indexer_scores -- lightning-indexer scores of every visible key
 * ("Inside a DSA layer: the lightning indexer"):
 *   scores[b][t][s] = sum_h w[b][t][h] * max(0, q_scale[b][t][h] * index_k_scale[row(b,s)]
 *                                             * <q8[b][t][h][:], index_k[row(b,s)][:]>)
 * for 0 <= s <= q_pos[b][t]; the entries q_pos[b][t] < s <= max_t q_pos[b][t]
 * are written as -infinity; entries beyond are not touched.
 * e4m3 products, fp32 accumulation on the tensor cores.  Needs scores_stride
 * >= Lmax >= max q_pos + 1, T <= DSA_MAX_T, q_scale and index_k_scale > 0.
 */
int dsa_indexer_scores(const void *q8, const float *q_scale, const float *w,
                       const dsa_kv_t *kv, const int32_t *q_pos, int B, int T,
                       int64_t Lmax, float *scores, int64_t scores_stride,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * dsa_index_produce -- the indexer's inputs for B x T new tokens ("Inside a
 * DSA layer: the lightning indexer": the indexer normalises its key, applies
 * RoPE, and rounds both query and key to fp8_e4m3; the section's figure names
 * LayerNorm, partial RoPE and FP8 quantisation; the same section gives the
 * attention block's partial RoPE on a third of each head and a rope base of
 * 10,000,000 on the sparse layers):
 *   key   y = LayerNorm(k_in[b][t]) (population variance, ln_eps, weight
 *         ln_w[128], bias ln_b[128]), then partial RoPE at p = q_pos[b][t];
 *         index_k[row(b, p)] = e4m3(y / s), index_k_scale[row(b, p)] = s,
 *         s = max|y| / 448 (1 for an all-zero y);
 *   query (when q_in is not NULL) every head of q_in[b][t] turned by the same
 *         partial RoPE at p; q8_out[b][t] = e4m3(y / s) with ONE scale s for
 *         the token's 16 heads, written to all 16 entries of q_scale_out[b][t].
 * Partial RoPE: dims i and i + rope_dim/2 (i < rope_dim/2) are rotated
 * together by the angle p * rope_base^(-2i / rope_dim) (x_i cos - x_{i+h}
 * sin, x_{i+h} cos + x_i sin); dims >= rope_dim pass unchanged.  rope_dim is
 * even, 0..128 (0.334 x 128 rounds down to 42).  e4m3 conversion: nearest
 * value, ties to the even code, saturating at +-448, taken in fp32.
 *   k_in   bf16 [B][T][128]          q_in     bf16 [B][T][16][128] or NULL
 *   q8_out uint8 [B][T][16][128]     q_scale_out float [B][T][16]
 *   kv     the index-key cache (index_k, index_k_scale and the layout) written
 *          at each token's position; a position outside it is flagged
 *          DSA_ERR_DEVICE_BAD_INDEX in the workspace and not written.
 * Workspace: dsa_workspace_size(DSA_OP_PRODUCE, ...) bytes (the status word).
 */
int dsa_index_produce(const void *k_in, const void *q_in, const float *ln_w, const float *ln_b, float ln_eps,
                      int rope_dim, double rope_base, const dsa_kv_t *kv, const int32_t *q_pos, int B, int T,
                      void *q8_out, float *q_scale_out, void *ws, size_t ws_bytes, void *stream);

/*
 * dsa_indexer_kl -- the indexer warm-up target and loss for B x T query
 * tokens ("Inside a DSA layer: the lightning indexer": the indexer is trained
 * first, alone, aligned to a full-attention reference by a KL objective; "2,122
 * tok/s, Zero Full-Attention Layers", "What's genuinely new": the converted
 * layers keep full attention and supervise the indexer through a KL loss).
 * For query (b, t) at p = q_pos[b][t], over its visible keys s = 0..p:
 *   P[s]  = (1/64) sum_h softmax_s(sm_scale * Q[b][t][h] . K[row(b,s)][h / (64/G)])
 *           (dense attention of each head, no sink, averaged over the heads)
 *   kl_out[b][t] = sum_s P[s] (ln P[s] - ln softmax_s(scores[b][t][s]))
 * target_out (float [B][T][target_stride], or NULL) receives P[0..p].
 * Q bf16 [B][T][64][192]; kv: the backbone keys (k, num_kv_heads, layout);
 * scores: the indexer's output for the same tokens (dsa_indexer_scores).
 * Logits on the tensor cores (bf16 operands, fp32 accumulation), softmax and
 * KL in fp32; every reduction in a fixed order (run-to-run identical).
 * Workspace: dsa_workspace_size(DSA_OP_KL, B, T, Lmax, 1, ...).
 */
int dsa_indexer_kl(const void *Q, const dsa_kv_t *kv, const float *scores, int64_t scores_stride,
                   const int32_t *q_pos, int B, int T, int64_t Lmax, float sm_scale, float *kl_out, float *target_out,
                   int64_t target_stride, void *ws, size_t ws_bytes, void *stream);

/*
 * dsa_topk_select -- for each query (b, t): the min(top_k, n) positions among
 * 0..n-1 (n = q_pos[b][t] + 1) with the largest scores, equal scores broken
 * toward the lower position, -0.0 equal to +0.0 ("What 'no full-attention
 * layers' means": argsort(...)[:, :top_k]).  idx[b][t][:] receives the
 * selected positions in increasing position order, padded with -1;
 * count[b][t] = min(top_k, n).  Scores must not be NaN.  1 <= top_k <=
 * DSA_MAX_TOPK.
 */
int dsa_topk_select(const float *scores, int64_t scores_stride, const int32_t *q_pos,
                    int B, int T, int64_t Lmax, int top_k, int32_t *idx, int32_t *count,
                    void *ws, size_t ws_bytes, void *stream);

/*
 * sparse_gqa_attn_decode -- softmax attention of each query head over the
 * selected key positions only ("Inside a DSA layer": the main heads gather
 * and attend to the selected K/V), grouped-query with contiguous head groups
 * (head h reads KV head h / (64 / G)), and an optional per-head sink logit in
 * the denominator:
 *   s_i = sm_scale * Q[h] . K[row(b, idx_i)][g]
 *   O[h] = sum_i e^{s_i} V[row(b, idx_i)][g] / (sum_i e^{s_i} + e^{sink[h]})
 * idx [B][T][top_k] (first count[b][t] entries used; each must satisfy
 * 0 <= idx <= q_pos is NOT required, only 0 <= idx < capacity of the
 * sequence).  sink may be NULL (no sink term); lse may be NULL.
 * A query with count == 0 and no sink gets O = 0 and lse = -inf.
 */
int sparse_gqa_attn_decode(const void *Q, const dsa_kv_t *kv, const int32_t *idx,
                           const int32_t *count, int B, int T, int top_k,
                           const float *sink, float sm_scale, void *O, float *lse,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * swa_attn_decode -- the same attention over the implicit contiguous key set
 * {max(0, p - window + 1) .. p}, p = q_pos[b][t] ("What 'no full-attention
 * layers' means": keys with query_offset - key_offset >= window are masked).
 * 1 <= window <= DSA_MAX_TOPK.
 */
int swa_attn_decode(const void *Q, const dsa_kv_t *kv, const int32_t *q_pos, int B, int T,
                    int window, const float *sink, float sm_scale, void *O, float *lse,
                    void *ws, size_t ws_bytes, void *stream);

/*
 * dsa_layer_decode -- one DSA decode layer-step: dsa_indexer_scores, then
 * dsa_topk_select, then sparse_gqa_attn_decode, enqueued back to back on
 * `stream` with the scores and the selection kept in the workspace.
 * idx_out (int32 [B][T][top_k]) and count_out (int32 [B][T]) are optional
 * copies of the selection (NULL = not wanted).
 * stage_events: NULL, or an array of 5 cudaEvent_t recorded on `stream`
 * before the indexer, before the selection, before the attention, before the
 * combine and at the end (for per-stage timing); NULL entries are skipped.
 * Event 0 is recorded after the host-side preparation, right before the first
 * kernel.  When the step runs as one fused kernel (B*T <= 16), events 1-4 are
 * all recorded after it.
 */
int dsa_layer_decode(const void *q8, const float *q_scale, const float *w, const void *Q,
                     const dsa_kv_t *kv, const int32_t *q_pos, int B, int T, int64_t Lmax,
                     int top_k, const float *sink, float sm_scale, void *O, float *lse,
                     int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes,
                     void *stream, void *const *stage_events);

/*
 * dsa_layer_chain -- a sequence of decode layer-steps enqueued as one chain,
 * the way a layer stack runs them ("The runtime is the actual claim": the
 * kernels of dependent steps chained with programmatic dependent launch).
 * Step i is exactly the call its kind names -- swa_attn_decode (window =
 * top_k) or dsa_layer_decode -- with the step's arguments, in order on
 * `stream`, and the outputs are bit-identical to making those calls one by
 * one.  The difference is the launch: every kernel that is not a
 * cooperative launch is enqueued as a programmatic dependent of the kernel
 * before it, so it is scheduled while that kernel finishes and waits for its
 * completion (and memory) before it touches anything; the cooperative
 * kernels (the fused layer-step, a multi-CTA selection) keep plain stream
 * order.  Every step is checked before anything is enqueued: an error in any
 * step returns before the first launch.  Steps may share a workspace (they
 * run one after another) or have their own.
 */
#define DSA_STEP_SWA 1
#define DSA_STEP_DSA 2
typedef struct dsa_layer_step {
    int32_t          kind;        /* DSA_STEP_SWA or DSA_STEP_DSA */
    int32_t          B, T;
    int32_t          top_k;       /* DSA: top_k; SWA: the window */
    int64_t          Lmax;        /* DSA: as for dsa_layer_decode */
    const void      *q8;          /* DSA only: index queries, scales, head weights */
    const float     *q_scale;
    const float     *w;
    const void      *Q;
    const dsa_kv_t  *kv;
    const int32_t   *q_pos;
    const float     *sink;        /* or NULL */
    float            sm_scale;
    int32_t          reserved;
    void            *O;
    float           *lse;         /* or NULL */
    int32_t         *idx_out;     /* DSA, or NULL */
    int32_t         *count_out;   /* DSA, or NULL */
    void            *ws;
    size_t           ws_bytes;
} dsa_layer_step_t;
int dsa_layer_chain(const dsa_layer_step_t *steps, int n_steps, void *stream);

/*
 * Context-sharded decode: the DSA layer-step with each sequence's context
 * split over n_ranks ranks, rank r holding the contiguous slice of positions
 * [shard_offset, shard_offset + shard_len) in its own caches (a design of this
 * library for multi-GPU decode; the pages describe the training system's
 * sequence parallelism -- Ulysses for the DSA layers, "2,122 tok/s, Zero
 * Full-Attention Layers", "What's genuinely new" -- not a decode split).
 * Per rank, with the exchanges done by the caller's collectives:
 *   1. dsa_shard_positions: q_pos_local = min(q_pos - shard_offset, shard_len - 1)
 *      (every query must sit at or after the slice's start; one before it is
 *      flagged DSA_ERR_DEVICE_BAD_INDEX in the workspace status word);
 *   2. dsa_indexer_scores + dsa_topk_select on the slice with q_pos_local;
 *   3. dsa_shard_candidates: the local selection as (score, global position)
 *      pairs, cand_score float [B][T][top_k] / cand_pos int32 [B][T][top_k],
 *      (-inf, -1) past the local count;
 *   4. all-gather of the pairs in rank order -> [n_ranks][B][T][top_k];
 *   5. dsa_shard_merge: the global top_k of every row (score descending, ties
 *      to the lower position -- the one-GPU rule) in position order into
 *      idx_out / count_out, and this rank's share as local positions,
 *      compacted and -1 padded, into local_idx / local_count (optional);
 *   6. sparse_gqa_attn_decode over (local_idx, local_count) with sink = NULL,
 *      giving O_r and lse_r (lse_r = -inf for a rank with no share);
 *   7. all-gather of (O_r, lse_r) in rank order;
 *   8. dsa_shard_combine: O = sum_r e^{lse_r - LSE} O_r with
 *      LSE = ln(sum_r e^{lse_r} + e^{sink}), the sink added once (sink may be
 *      NULL); lse receives LSE.
 * The merged selection equals the one-GPU selection over the whole context
 * bit for bit; the output equals the one-GPU output within the attention
 * tolerance (the sum is split by owner).  n_ranks 1..8.  These calls need no
 * workspace except dsa_shard_positions (DSA_OP_PRODUCE, the status word).
 */
int dsa_shard_positions(const int32_t *q_pos, int B, int T, int64_t shard_offset, int64_t shard_len,
                        int32_t *q_pos_local, void *ws, size_t ws_bytes, void *stream);
int dsa_shard_candidates(const float *scores, int64_t scores_stride, const int32_t *idx, int B, int T, int top_k,
                         int64_t shard_offset, float *cand_score, int32_t *cand_pos, void *stream);
int dsa_shard_merge(const float *cand_score, const int32_t *cand_pos, int n_ranks, int B, int T, int top_k,
                    int64_t shard_offset, int64_t shard_len, int32_t *idx_out, int32_t *count_out,
                    int32_t *local_idx, int32_t *local_count, void *stream);
int dsa_shard_combine(const void *O_all, const float *lse_all, int n_ranks, int B, int T, const float *sink, void *O,
                      float *lse, void *stream);

/*
 * dsa_prefill -- the DSA layer for NQ query tokens of ONE sequence (a
 * prefill chunk, or any block of queries over a shared cache): for each query
 * token t at position q_pos[t], exactly the decode layer-step -- indexer
 * scores over its visible keys 0..q_pos[t] (causal), the top_k selection, the
 * sparse GQA attention with the sink -- as dsa_layer_decode computes it, bit
 * for bit ("What 'no full-attention layers' means": every DSA query keeps its
 * own top 2,048 of the keys it may see).
 *   q8       e4m3 [NQ][16][128]      q_scale, w  f32 [NQ][16]
 *   Q        bf16 [NQ][64][192]      q_pos       int32 [NQ], each < Lmax
 *   kv       the sequence's caches (B = 1), as for dsa_layer_decode
 *   O        bf16 [NQ][64][128]      lse         f32 [NQ][64] or NULL
 *   idx_out  int32 [NQ][top_k] or NULL; count_out int32 [NQ] or NULL
 * When NQ is a multiple of 16 (>= 64), the cache is contiguous or paged with
 * pages of at most 256 positions, and Lmax >= 4,096, the indexer runs as one
 * fp8 contraction of all NQ x 16 query heads against the keys on the tensor
 * cores, keeping for each token only the keys above a threshold estimated
 * from a sample of the keys (every 64th page), never the NQ x Lmax score
 * matrix; each token's exact top_k is then taken from its candidates, and the
 * attention runs over all tokens.  A token whose candidates turn out not to
 * hold its selection (heavy ties, an unusual score distribution) is
 * recomputed by the decode layer-step; this path reads that (usually empty)
 * list back to the host, so the call synchronises `stream` once and cannot be
 * captured in a CUDA graph.  Other shapes run DSA_MAX_T tokens at a time
 * (one dsa_layer_decode per block, asynchronous).
 * Workspace: dsa_workspace_size(DSA_OP_PREFILL, 1, NQ, Lmax, top_k) (about
 * 1.4 GB for 8,192 tokens at 1,048,576 context: the sample's scores and the
 * candidate lists).  Errors as for dsa_layer_decode.
 */
int dsa_prefill(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                const int32_t *q_pos, int NQ, int64_t Lmax, int top_k, const float *sink, float sm_scale,
                void *O, float *lse, int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes,
                void *stream);

/*
 * dsa_topk_select_noalloc -- the selection of dsa_topk_select for callers
 * that cannot allocate device memory and so cannot provide a workspace: a
 * framework that owns every device allocation and refuses new ones after it
 * starts, a latency-critical loop that must never reach the allocator, a
 * plug-in handed only its input and output buffers.  (The pages have no
 * counterpart; this is an interface convenience of this library.)
 *
 * Same arguments and results as dsa_topk_select, without ws / ws_bytes.  The
 * scratch is a 2 MiB array in device memory declared by the library itself;
 * every GPU that loads the library holds it until the process exits.  A call
 * whose scratch need exceeds it returns DSA_ERR_UNSUPPORTED_SHAPE with a
 * message (use dsa_topk_select with a workspace then); on a 148-SM B200 the
 * largest fixed need is about 1.5 MB (74 query rows split two CTAs each) and
 * the selection's candidate list is shortened to the room left (down to none,
 * which exchanges every digit instead), so every shape dsa_topk_select
 * accepts fits.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents; each call clears the part that must start at zero
 *     (cudaMemsetAsync on `stream`) before its kernel.  Calls that may overlap
 *     on the GPU (different streams, or concurrent host threads) race on the
 *     array: serialise them.
 *   - Device-side status (bad positions, a bounded wait running out) is
 *     recorded in the array but not reported by this entry point.
 */
int dsa_topk_select_noalloc(const float *scores, int64_t scores_stride, const int32_t *q_pos, int B, int T,
                            int64_t Lmax, int top_k, int32_t *idx, int32_t *count, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
