// fused.cu -- the whole DSA decode layer-step in one persistent, cooperative
// kernel: lightning indexer -> top-k selection -> split-KV sparse attention ->
// split combine, with grid-wide barriers between the phases and no launch in
// between.  ("Naive-N0.5-Flash: no full-attention layers, and a runtime built
// by AI", section "The runtime is the actual claim", describes a DSA layer run
// as one cooperative kernel on 148 CTAs; this is this library's own design of
// that idea for B200, built from the same device code as the standalone
// kernels.)
//
// Grid: one CTA per SM (as the indexer), 640 threads each, all co-resident
// (cooperative launch).
//   phase 1  indexer body (indexer_impl.cuh); scores to the workspace and,
//            for up to kMaxHistRows rows, each CTA's histogram of its scores
//            (bits 30..20 of the non-negative keys, plus a count of the
//            negative ones) added into the rows' global histograms;
//   phase 2  selection (topk_impl.cuh), each query row shared by
//            C = grid / rows CTAs: the one-barrier path from that histogram
//            where the row qualifies, the general path otherwise;
//   phase 3  attention units (attention_impl.cuh): four teams of four warps
//            per CTA, one (query, KV head, 64-key split) unit per team at a
//            time, reading the -1-padded selection; the four other warps
//            clear the selection scratch for the next call;
//   phase 4  combine: one CTA per (query, head).
#include <algorithm>
#include <mutex>

#include "attention_impl.cuh"
#include "indexer_impl.cuh"
#include "kernels.h"
#include "topk_impl.cuh"

namespace dsa {
namespace fused {

constexpr int kThreads = indexer::kThreads;   // 640
constexpr int kWarps = kThreads / 32;
constexpr int kTeams = 4;                     // attention teams of 4 warps (named barriers 1..4)
constexpr int kMaxRows = 16;                  // B * T handled by the fused path
constexpr int kMaxHistRows = 8;               // rows whose first histogram the indexer builds
constexpr int kUnitBar = 9;                   // named barrier of the attention teams of a CTA unit

static_assert(kTeams * 4 < kWarps, "the attention teams must leave warps free in the CTA");

struct Params {
    indexer::Params ix;
    topk::Params tk;
    attn::Params at;
    const float *sink;
    __nv_bfloat16 *O;
    float *lse;
    uint32_t *grid_bar;   // [0] arrivals, [1] exits
    BarrierCfg bar;       // time limit (and injected extra arrivals) of the grid barriers
    int rows;             // B * T
    int C;                // CTAs per row in the selection phase
    int hist_ready;
};

__host__ __device__ constexpr size_t smem_align(size_t x) { return (x + 127) & ~size_t(127); }

__global__ void __launch_bounds__(kThreads, 1)
dsa_layer_fused_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_ks,
                       const __grid_constant__ CUtensorMap tmap_q, const Params fp) {
    // the dynamic buffer is aligned by hand (its 1 KB slack is part of the budget), so the
    // static shared memory of this kernel stays a few bytes
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // aligned by an offset from the array itself, so the compiler keeps the shared address space
    uint8_t *smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    __shared__ uint32_t sync_flag;
    pdl_begin();
    const uint32_t G = gridDim.x;
    uint32_t *status = fp.ix.status;
    const uint32_t status_at_entry = load_status(status);

    // ---- phase 1: indexer
    indexer::run_indexer(&tmap_k, &tmap_ks, &tmap_q, fp.ix, smem, blockIdx.x, G);
    if (status_at_entry & kNeedsInitBit) {   // the cross-CTA scratch is not in its clean state
        if (threadIdx.x == 0) flag_timeout(status);
        return;
    }
    if (!grid_sync(fp.grid_bar, 1 * G, fp.bar, status, &sync_flag)) return;

    // ---- phase 2: selection (candidate runs when the indexer built the first histogram;
    //      the round-by-round path otherwise, or when the candidates would not fit)
    if ((int)blockIdx.x < fp.rows * fp.C) {
        auto *sh = reinterpret_cast<topk::Shared<kThreads> *>(smem);
        uint32_t *cache = reinterpret_cast<uint32_t *>(smem + smem_align(sizeof(topk::Shared<kThreads>)));
        const int row = blockIdx.x / fp.C, c = blockIdx.x % fp.C;
        bool done = false;
        if (fp.hist_ready && fp.C > 1) done = topk::select_row_hist<kThreads>(fp.tk, sh, cache, row, c, fp.C);
        if (!done) topk::select_row<kThreads>(fp.tk, sh, cache, row, c, fp.C, true);
    }
    if (!grid_sync(fp.grid_bar, 2 * G, fp.bar, status, &sync_flag)) return;

    // ---- phase 3: attention units (one team each, the CTA's teams on four
    //      units at once; or CTA units of n_teams merged teams)
    {
        const int nt = fp.at.n_teams;
        const attn::TeamSmem teams{smem, (uint32_t)smem_align(sizeof(attn::Smem))};
        const int G_kv = fp.at.G, splits = fp.at.splits;
        const int units = fp.rows * G_kv * splits;
        if ((int)threadIdx.x < kTeams * 128) {
            if (nt == 1) {
                const int tm = threadIdx.x >> 7;
                for (int u = blockIdx.x + tm * G; u < units; u += kTeams * G) {
                    const int split = u % splits, g = (u / splits) % G_kv, bt = u / (splits * G_kv);
                    attn::team_unit(fp.at, teams[tm], split, g, bt, threadIdx.x & 127, 1 + tm, fp.sink, fp.O,
                                    fp.lse);
                }
            } else if ((int)threadIdx.x < nt * 128) {
                for (int u = blockIdx.x; u < units; u += G) {
                    const int split = u % splits, g = (u / splits) % G_kv, bt = u / (splits * G_kv);
                    attn::cta_unit(fp.at, teams, split, g, bt, 1, kUnitBar, fp.sink, fp.O, fp.lse);
                }
            }
        } else if ((int)threadIdx.x >= kTeams * 128 && (int)blockIdx.x < fp.rows * fp.C && (fp.C > 1 || fp.hist_ready)) {
            // the warps outside the teams clear the selection scratch for the next call
            constexpr int kFree = kThreads - kTeams * 128;
            topk::clear_row_share(fp.tk, blockIdx.x / fp.C, blockIdx.x % fp.C, fp.C, fp.hist_ready != 0,
                                  threadIdx.x - kTeams * 128, kFree);
        }
    }
    if (!grid_sync(fp.grid_bar, 3 * G, fp.bar, status, &sync_flag)) return;
    if ((int)blockIdx.x < fp.rows * fp.C && blockIdx.x % fp.C == 0) topk::reset_row_ctl(fp.tk, blockIdx.x / fp.C, fp.C);

    // ---- phase 4: combine of the units, one CTA per (query, head)
    if (fp.at.splits > 1)
        for (int gw = blockIdx.x; gw < fp.rows * DSA_Q_HEADS; gw += G)
            attn::combine_row_cta<kThreads>(fp.at.part_o, fp.at.part_ml, gw, fp.at.splits, fp.sink, fp.O, fp.lse,
                                            reinterpret_cast<float *>(smem));

    // ---- the last CTA out resets the grid barrier for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(fp.grid_bar + 1, 1u) == G - 1) {
            atomicExch(fp.grid_bar, 0u);
            atomicExch(fp.grid_bar + 1, 0u);
        }
    }
}

}  // namespace fused

// Largest dynamic shared memory of the fused kernel: half an SM, minus room
// for its few bytes of static shared memory.
static size_t fused_smem_budget() {
    // one CTA per SM; leave room for the kernel's few bytes of static shared memory
    return device_info().smem_optin - 1024;
}

int plan_fused(int B, int T, int64_t Lmax, int top_k, FusedPlan *plan) {
    using namespace fused;
    const DeviceInfo &dev = device_info();
    plan->ok = false;
    const int rows = B * T;
    if (dev.num_sms <= 0 || rows > kMaxRows) return DSA_OK;
    const int64_t max_tiles = (int64_t)B * ((Lmax + indexer::kTile - 1) / indexer::kTile);
    // all CTAs must be resident at once (the phases wait on each other): as many as fit
    // (the occupancy query is made once per device)
    static std::mutex mu;
    static int per_sm_cache[64];
    static bool known[64] = {};
    int dev_id = -1;
    cudaError_t e = cudaGetDevice(&dev_id);
    if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) return cuda_fail(e, "cudaGetDevice");
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!known[dev_id]) {
            if (int rc = ensure_smem_limit((const void *)dsa_layer_fused_kernel, fused_smem_budget(),
                                           "cudaFuncSetAttribute(fused)"))
                return rc;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_cache[dev_id], dsa_layer_fused_kernel, kThreads,
                                                              fused_smem_budget());
            if (e != cudaSuccess) return cuda_fail(e, "occupancy of the fused kernel");
            known[dev_id] = true;
        }
        per_sm = per_sm_cache[dev_id];
    }
    per_sm = std::min(per_sm, 1);
    if (per_sm < 1 || rows > per_sm * dev.num_sms) return DSA_OK;
    // every CTA takes part in every phase: at least one CTA per row for the selection
    const int grid = (int)std::max<int64_t>(
        rows, std::min<int64_t>((int64_t)dev.num_sms * per_sm, max_tiles));
    plan->grid = grid;
    plan->rows = rows;
    plan->C = std::max(1, grid / rows);
    plan->scratch_bytes = (size_t)rows * topk::scratch_words(plan->C, topk::kListCap, true) * 4 + 256;   // + grid barrier words
    plan->ok = true;
    return DSA_OK;
}

int launch_fused(const FusedPlan &plan, const IndexerArgs &ia, const AttnArgs &aa, int top_k, int32_t *idx,
                 int32_t *count, uint32_t *scratch, cudaStream_t stream,
                 void *start_event) {
    using namespace fused;
    const size_t budget = fused_smem_budget();
    uint32_t *row_scratch = scratch + 64;   // the first 256 bytes hold the grid barrier words
    const int row_words = topk::scratch_words(plan.C, topk::kListCap, true);

    // indexer phase, with the first histogram when the rows' histograms fit
    IndexerLaunch L;
    int hist_rows = plan.rows <= kMaxHistRows ? plan.rows : 0;
    int rc = prepare_indexer(ia, hist_rows, row_words, row_scratch + topk::histi_base(plan.C, topk::kListCap), budget, &L);
    if (rc == DSA_OK && hist_rows && L.p.stages < 3) hist_rows = 0;   // keep the stream at least 3 stages deep
    if (rc != DSA_OK || hist_rows == 0) {
        hist_rows = 0;
        if ((rc = prepare_indexer(ia, 0, 0, nullptr, budget, &L))) return rc;
    }
    // the indexer body spreads its tiles over however many CTAs run it

    Params fp;
    fp.ix = L.p;
    fp.at = attn::make_params(aa);
    fp.sink = aa.sink;
    fp.O = aa.O;
    fp.lse = aa.lse;
    fp.grid_bar = scratch;
    fp.bar = barrier_cfg();
    fp.rows = plan.rows;
    fp.C = plan.C;
    fp.hist_ready = hist_rows > 0;

    // selection phase: same parameters as the standalone selection
    const size_t attn_smem = kTeams * smem_align(sizeof(attn::Smem));
    const size_t top_fixed = smem_align(sizeof(topk::Shared<kThreads>));
    const size_t smem = std::max({L.smem, attn_smem + 1024, top_fixed + 1024 + 4096});
    if (smem > budget) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "fused kernel shared memory does not fit");
    topk::Params &tp = fp.tk;
    tp.scores = ia.scores;
    tp.stride = ia.scores_stride;
    tp.q_pos = ia.q_pos;
    tp.rows = plan.rows;
    tp.K = top_k;
    tp.C = plan.C;
    tp.idx = idx;
    tp.count = count;
    tp.scratch = row_scratch;
    tp.scratch_row_words = row_words;
    tp.status = ia.status;
    {   // shared memory after the fixed part: the CTA's slice of keys, then the candidate list
        const int64_t avail = (int64_t)(smem - 1024 - top_fixed) / 4;
        const int64_t chunk = ((ia.Lmax + plan.C - 1) / plan.C + 3) & ~int64_t(3);
        const int64_t cand = std::min<int64_t>(topk::kCandCap, avail / 4) / kWarps * kWarps;
        const int64_t rest = avail - 2 * cand;
        int64_t list = std::min<int64_t>(topk::kListCap, std::max<int64_t>(0, (rest - chunk) / 2));
        if (list < 1024) list = std::min<int64_t>(topk::kListCap, rest / 4);   // slices too long to cache
        tp.smem_list = (int)list;
        tp.cand_cap = (int)cand;
        tp.cache_keys = (int)(rest - 2 * list);
    }
    tp.list_cap = topk::kListCap;
    tp.Lmax = ia.Lmax;
    tp.bar = fp.bar;

    if ((rc = ensure_smem_limit((const void *)dsa_layer_fused_kernel, smem, "cudaFuncSetAttribute(fused)"))) return rc;
    cudaError_t e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // the phases wait on every CTA
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (start_event) {   // recorded after the host-side preparation, right before the launch
        e = cudaEventRecord(static_cast<cudaEvent_t>(start_event), stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    e = cudaLaunchKernelEx(&cfg, dsa_layer_fused_kernel, L.tmap_k, L.tmap_ks, L.tmap_q, fp);
    if (e != cudaSuccess) return cuda_fail(e, "fused layer-step launch");
    return DSA_OK;
}

}  // namespace dsa
