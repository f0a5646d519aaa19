// kernels.h -- host-side launchers of the libdsa kernels (internal to the
// library; the public boundary is include/dsa.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// Device properties the launchers size their grids with (cached per device).
struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    size_t smem_optin = 0;
};
const DeviceInfo &device_info();

// Raises a kernel's dynamic shared memory limit to at least `bytes` on the
// current device; the attribute call is made only when the cached limit is
// lower (it is per device and per kernel, and costs a driver call).
int ensure_smem_limit(const void *kernel, size_t bytes, const char *what);

// Launches made from this host thread while a dsa_layer_chain call is
// enqueueing carry the programmatic-stream-serialization attribute (each
// kernel may be scheduled before the previous one ends; pdl_begin orders
// their memory).
bool pdl_launches();
void set_pdl_launches(bool on);

// A plain (non-cooperative) launch, chained when pdl_launches().
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_as(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args... args);
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args... args) {
    return launch_kernel_as(pdl_launches(), kernel, grid, block, smem, stream, args...);
}

// As launch_kernel, with programmatic dependent launch when `pdl` (every
// kernel of this library waits for its predecessor at its first instruction).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_as(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Sets the thread-local error message and returns `code`.
int fail(int code, const char *fmt, ...);
// Converts a CUDA runtime error into DSA_ERR_CUDA with a message.
int cuda_fail(cudaError_t e, const char *what);

// ---------------------------------------------------------------- indexer
struct IndexerArgs {
    const uint8_t *q8;
    const float *q_scale;
    const float *w;
    const dsa_kv_t *kv;
    const int32_t *q_pos;
    int B, T;
    int64_t Lmax;
    float *scores;
    int64_t scores_stride;
    uint32_t *status;
};
int launch_indexer(const IndexerArgs &a, cudaStream_t stream);

namespace indexer { struct Params; }
// Tiled tensor map (cached per device, base, shape and box; see indexer.cu).
int make_tensor_map(const char *what, CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base,
                    const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz);
// Everything a launch of the indexer body needs: tensor maps, parameters,
// dynamic shared memory and grid (one CTA per SM, two pipelines per CTA).  hist_rows > 0 adds each
// CTA's histogram of the visible scores (see indexer::kHistWords) into hist_global.
struct IndexerLaunch;
int prepare_indexer(const IndexerArgs &a, int hist_rows, int hist_row_words, uint32_t *hist_global,
                    size_t smem_budget, IndexerLaunch *out);

// ----------------------------------------------------------------- top-k
struct TopkPlan {
    int rows = 0;          // B * T
    int ctas_per_row = 1;  // C
    int threads = 512;
    int cache_keys = 0;    // keys cached in shared memory per CTA
    int list_cap = 0;      // candidate-list entries per row in the scratch
    int smem_list = 0;     // candidate-list entries that fit in shared memory
    int cand_cap = 0;      // per-warp candidate entries in shared memory, all warps together
    int64_t Lmax = 0;      // positions held by each scores row
    bool var_c = false;    // CTAs per row follow the rows' lengths (ctas_per_row is then the most a row gets)
    size_t smem = 0;
    size_t scratch_bytes = 0;  // cross-CTA scratch (only when C > 1)
};
// max_scratch_bytes bounds scratch_bytes by shortening the candidate list
// (down to none: the selection then exchanges every digit).
int plan_topk(int B, int T, int64_t Lmax, int top_k, TopkPlan *plan, size_t max_scratch_bytes = SIZE_MAX);
int launch_topk(const TopkPlan &plan, const float *scores, int64_t stride, const int32_t *q_pos,
                int top_k, int32_t *idx, int32_t *count, uint32_t *scratch, uint32_t *status,
                cudaStream_t stream, float *kth = nullptr);

// ------------------------------------------------------ index-K / index-Q producer
struct ProduceArgs {
    const __nv_bfloat16 *k_in;   // [B*T][128]
    const __nv_bfloat16 *q_in;   // [B*T][16][128] or null
    const float *ln_w, *ln_b;
    float ln_eps;
    int rope_dim;
    double rope_base;
    const dsa_kv_t *kv;
    const int32_t *q_pos;
    int B, T;
    uint8_t *q8;
    float *q_scale;
    uint32_t *status;
};
int launch_index_produce(const ProduceArgs &a, cudaStream_t stream);

// ------------------------------------------------------ indexer warm-up KL
struct KlArgs {
    const __nv_bfloat16 *Q;
    const dsa_kv_t *kv;
    const float *scores;
    int64_t scores_stride;
    const int32_t *q_pos;
    int B, T;
    int64_t Lmax;
    float sm_scale;
    float *kl_out;
    float *target;
    int64_t target_stride;
    void *scratch;
    uint32_t *status;
};
size_t kl_workspace_bytes(int B, int T, int64_t Lmax);
int launch_indexer_kl(const KlArgs &a, cudaStream_t stream);

// ------------------------------------------------ chunked prefill (prefill.cu)
struct PrefillPlan {
    bool ok = false;
    int NQ = 0, K = 0, nblocks = 0, B_rep = 0, s = 0, max_ps = 0, cap = 0, attn_chunk = 0;
    int64_t Lmax = 0, Ls_cap = 0;
    TopkPlan tp;
    size_t topk_scratch = 0, sample_table = 0, sample_pos = 0, sample_scores = 0, sample_idx = 0, sample_cnt = 0,
           thr = 0, meta = 0, block_max = 0, cand_cnt = 0, cand = 0, idx = 0, count = 0, redo_n = 0, redo = 0,
           part_o = 0, part_ml = 0, total = 0;
};
struct PrefillArgs {
    const uint8_t *q8;
    const float *q_scale, *w;
    const __nv_bfloat16 *Q;
    const dsa_kv_t *kv;
    const int32_t *q_pos;
    int64_t Lmax;
    const float *sink;
    float sm_scale;
    __nv_bfloat16 *O;
    float *lse;
    int32_t *idx_out, *count_out;
    uint32_t *status;
};
int plan_prefill_capture(int NQ, int64_t Lmax, int top_k, PrefillPlan *plan);
// Runs the four stages; the tokens whose candidates did not hold their
// selection (written with count 0) are listed in redo_host[0 .. *n_redo).
// Synchronises the stream (to read that list).
int run_prefill_capture(const PrefillPlan &plan, const PrefillArgs &a, uint8_t *ws, cudaStream_t s,
                        int32_t *redo_host, int *n_redo);

// -------------------------------------------------- context-sharded decode
int launch_shard_positions(const int32_t *q_pos, int rows, int64_t offset, int64_t len, int32_t *q_local,
                           uint32_t *bad, cudaStream_t stream);
int launch_shard_candidates(const float *scores, int64_t stride, const int32_t *idx, int K, int rows, int64_t offset,
                            float *cand_score, int32_t *cand_pos, cudaStream_t stream);
int launch_shard_merge(const float *cand_score, const int32_t *cand_pos, int N, int K, int rows, int64_t rank_offset,
                       int64_t rank_len, int32_t *idx_out, int32_t *count_out, int32_t *local_idx,
                       int32_t *local_count, cudaStream_t stream);
int launch_shard_combine(const __nv_bfloat16 *O_all, const float *lse_all, int N, int rows, const float *sink,
                         __nv_bfloat16 *O, float *lse, cudaStream_t stream);

// ------------------------------------------------------------- attention
constexpr int kAttnChunk = 64;   // keys per team chunk (one team of 4 warps)
constexpr int kAttnMaxTeams = 4;
// Team chunks per CTA unit, and CTA units per (query, KV head), for a key set
// of at most max_keys keys: units of up to 256 keys.
// Teams of 64 keys per attention unit: up to kAttnMaxTeams teams merged in
// one CTA unit for a key set of at most 256 (one unit per query and KV head,
// no combine: the sliding window); a single team per unit above, so that a
// top-k selection spreads over one unit per 64 keys (at most 32 for
// DSA_MAX_TOPK) and every SM gathers a share.
inline int attn_teams(int max_keys) {
    const int c = (max_keys + kAttnChunk - 1) / kAttnChunk;
    if (c > kAttnMaxTeams) return 1;
    return c > 0 ? c : 1;
}
inline int attn_splits(int max_keys) {
    const int u = kAttnChunk * attn_teams(max_keys);
    return (max_keys + u - 1) / u;
}
struct AttnArgs {
    const __nv_bfloat16 *Q;
    const dsa_kv_t *kv;
    const int32_t *idx;     // sparse: [B*T][idx_stride]; NULL for the sliding window
    const int32_t *count;   // sparse: [B*T]
    int idx_stride;
    const int32_t *q_pos;   // sliding window: [B*T]
    int window;
    int B, T;
    int max_keys;           // top_k or window: bounds the number of splits
    const float *sink;
    float sm_scale;
    __nv_bfloat16 *O;
    float *lse;
    float *part_o;          // [B*T][64][splits][128]
    float *part_ml;         // [B*T][64][splits][2]
    uint32_t *status;
    void *mid_event = nullptr;  // optional cudaEvent_t recorded between the gather and the combine
    int padded = 0;             // idx rows full length, -1 past the selection (count not read)
};
size_t attn_partial_bytes(int B, int T, int max_keys);
int launch_attention(const AttnArgs &a, cudaStream_t stream);

// --------------------------------------------------------- fused layer-step
struct FusedPlan {
    bool ok = false;            // false: use the separate kernels
    int grid = 0;               // CTAs (one per SM)
    int rows = 0;               // B * T
    int C = 1;                  // CTAs per row in the selection phase
    size_t scratch_bytes = 0;   // grid barrier words + per-row selection scratch
};
int plan_fused(int B, int T, int64_t Lmax, int top_k, FusedPlan *plan);

// ------------------------------------------- layer-step with candidate capture
// The fused layer-step for B * T <= 4 rows of long contexts (capture.cu): the
// key stream samples the scores and keeps every key above a threshold in
// position-ordered candidate lists, so the selection needs one grid barrier.
struct CapturePlan {
    bool ok = false;            // false: use the fused or the separate kernels
    int grid = 0;
    int rows = 0;
    int C = 1;                  // CTAs per row
    int NG = 0;                 // CTAs in the grid (segments of each row's list)
    // self-cleaning scratch (zero between calls): control words, sample and
    // candidate histograms, the fallback selection's scratch
    size_t ctl_off = 0, hist_off = 0, topk_off = 0, cand_hist_off = 0;
    size_t scratch_bytes = 0;
    // overwritten by every call (never assumed zero): the candidate segments
    // and their lengths, in a workspace region of their own
    size_t counts_off = 0, lists_off = 0;
    size_t data_bytes = 0;
};
int plan_capture(int B, int T, int64_t Lmax, int top_k, CapturePlan *plan);
int launch_capture(const CapturePlan &plan, const IndexerArgs &ia, const AttnArgs &aa, int top_k, int32_t *idx,
                   int32_t *count, uint8_t *scratch, uint8_t *data, cudaStream_t stream,
                   void *start_event = nullptr);
int launch_fused(const FusedPlan &plan, const IndexerArgs &ia, const AttnArgs &aa, int top_k, int32_t *idx,
                 int32_t *count, uint32_t *scratch, cudaStream_t stream,
                 void *start_event = nullptr);


}  // namespace dsa
