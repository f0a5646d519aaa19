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
    size_t smem = 0;
    size_t scratch_bytes = 0;  // cross-CTA scratch (only when C > 1)
};
// max_scratch_bytes bounds scratch_bytes by shortening the candidate list
// (down to none: the selection then exchanges every digit).
int plan_topk(int B, int T, int64_t Lmax, int top_k, TopkPlan *plan, size_t max_scratch_bytes = SIZE_MAX);
int launch_topk(const TopkPlan &plan, const float *scores, int64_t stride, const int32_t *q_pos,
                int top_k, int32_t *idx, int32_t *count, uint32_t *scratch, uint32_t *status,
                cudaStream_t stream);

// ------------------------------------------------------------- attention
constexpr int kAttnChunk = 64;   // keys per split
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
int launch_fused(const FusedPlan &plan, const IndexerArgs &ia, const AttnArgs &aa, int top_k, int32_t *idx,
                 int32_t *count, uint32_t *scratch, cudaStream_t stream,
                 void *start_event = nullptr);


}  // namespace dsa
