// indexer_impl.cuh -- streaming lightning indexer on the 5th-generation
// tensor cores (device code shared by the standalone indexer kernel and the
// fused layer-step kernel).
//
// Computes, for every visible key s of every query (b, t),
//   I[b,t,s] = sum_h w[b,t,h] * max(0, qs[b,t,h] * ks[s] * <q8[b,t,h], k8[s]>)
// ("Naive-N0.5-Flash: no full-attention layers, and a runtime built by AI",
// section "Inside a DSA layer: the lightning indexer": relu(q k^T) per index
// head in fp8_e4m3, combined across the 16 heads by a learned weight).
// Because the scales are positive, relu(qs * ks * x) = qs * ks * relu(x), so
// the kernel takes the raw e4m3 dot products from the tensor cores and applies
// the scales in the epilogue: I = ks * sum_h (w_h qs_h) * relu(dot_h).
//
// Design (persistent, one CTA per SM, two independent pipelines per CTA,
// warp-specialised).  One TMA pipeline per SM does not reach the SM's share
// of HBM bandwidth on B200 (measured: ~0.65 us per 16 KB tile); two do.  Each
// pipeline p owns half of the CTA's contiguous tile range and has
//   warp p        TMA producer: per 128-key tile, the e4m3 key tile
//                 [128 x 128 B] (128-byte swizzle) and the 128 fp32 key scales
//                 (plus the query block [16T x 128 B] when several sequences
//                 share the call; one sequence keeps its query block resident);
//   warp 2 + p    MMA issuer: D[128 keys x 16T] = K_tile[128 x 128] Q^T with
//                 four tcgen05.mma kind::f8f6f4 (K=32 each), fp32 in TMEM;
//   4 warps per epilogue group, GE groups, each group with its own TMEM
//                 accumulator and every GE-th tile of the pipeline:
//                 tcgen05.ld of one key row per thread, ReLU, per-head
//                 weighting, key scale, causal mask, coalesced fp32 store,
//                 optionally a histogram of the scores for the selection.
#pragma once

#include "common.cuh"

namespace dsa {
namespace indexer {

constexpr int kTile = 128;                // keys per tile = UMMA M
constexpr int kKeyBytes = DSA_INDEX_DIM;  // 128 e4m3 codes per key
constexpr int kPipes = 2;                 // independent load -> MMA -> epilogue pipelines per CTA
constexpr int kMaxGroups = 2;             // epilogue groups per pipeline (one TMEM accumulator each)
constexpr int kEpiWarps = 4;              // warps per epilogue group (one per TMEM lane quarter)
constexpr int kEpiWarp0 = 2 * kPipes;     // first epilogue warp
constexpr int kThreads = 32 * (kEpiWarp0 + kPipes * kMaxGroups * kEpiWarps);   // 640
constexpr int kMaxStages = 8;             // per pipeline
constexpr int kAccBufs = 4;               // at most this many TMEM accumulators per epilogue group (two or
                                          // more: the MMA of a group's next tiles runs while its epilogue
                                          // reads this one)
constexpr int kKsStageBytes = 1024;       // key-scale slots of one stage
// Score histogram for the selection: bits 30..20 of the order key of each
// non-negative score (2048 bins, eight per octave), and one bin (2048) that
// counts the negative scores; kHistWords words per row.
constexpr int kHistBins = 2048;
constexpr int kHistWords = 2052;

// Byte offset, inside a stage's key-scale area, of the scale of tile row r.
__host__ __device__ __forceinline__ int ks_slot_offset(int r, int R) {
    const int slot = (R * 4 + 127) & ~127;
    return (r / R) * slot + (r % R) * 4;
}

struct Params {
    const float *q_scale;
    const float *w;
    const int32_t *q_pos;
    const int32_t *block_table;
    int32_t max_pages;
    int32_t page_size;
    int64_t seq_stride;
    int64_t num_rows;
    int B, T;
    int64_t Lmax;
    float *scores;
    int64_t scores_stride;
    uint32_t *status;
    int stages;          // per pipeline
    int rows_per_load;   // R: rows per TMA box (128, or the page size when pages are smaller)
    int groups;          // epilogue groups per pipeline (1..kMaxGroups)
    int acc_bufs;        // TMEM accumulators per group (1..kAccBufs); kPipes * groups * acc_bufs * 16T <= 512
    // optional histogram of the visible scores (see kHistWords), added into
    // hist_global[row * hist_row_words + bin] for rows b * T + t < hist_rows;
    // hist_rows == 0 turns it off
    int hist_rows;
    int hist_row_words;
    uint32_t *hist_global;
    // one sequence: its query block is loaded once and stays resident, instead
    // of riding along with every key tile
    int q_resident;
};

struct __align__(8) Bars {
    uint64_t full[kPipes][kMaxStages];
    uint64_t empty[kPipes][kMaxStages];
    uint64_t tfull[kPipes][kMaxGroups][kAccBufs];
    uint64_t tempty[kPipes][kMaxGroups][kAccBufs];
    uint64_t mma_done[kPipes];
    uint64_t q_full;
};

// Shared memory carve-up (base aligned to 1024 bytes), S stages per pipeline:
//   [0, P*S*16K)        key tiles, stage (p, s) at (p*S + s)*16K
//   query blocks        one resident block, or one per stage
//   P*S * 1 KB          key scales: one 128-byte aligned slot per TMA box
//                       (tensor copies need 128-byte aligned destinations)
//   Bars, TMEM address, per-sequence tables, per-warp epilogue constants,
//   optional per-row score histograms
struct Layout {
    uint32_t k_off, q_off, ks_off, bar_off, tmem_off, len_off, tile_off, epi_off, hist_off, total;
    __host__ __device__ Layout(int S, int T, int B, int hist_rows = 0, bool q_resident = false) {
        const int stages = kPipes * S;
        k_off = 0;
        q_off = k_off + stages * kTile * kKeyBytes;
        ks_off = q_off + (q_resident ? 1 : stages) * 16 * T * kKeyBytes;
        bar_off = ks_off + stages * kKsStageBytes;
        tmem_off = bar_off + (uint32_t)sizeof(Bars);
        len_off = (tmem_off + 16 + 15) & ~15u;
        tile_off = len_off + 4 * (B + 1);
        tile_off = (tile_off + 15) & ~15u;
        epi_off = tile_off + 4 * (B + 1);
        epi_off = (epi_off + 15) & ~15u;
        // per epilogue warp: 16*T coefficients + T positions
        hist_off = epi_off + kPipes * kMaxGroups * kEpiWarps * (16 * T + T) * 4;
        total = hist_off + hist_rows * kHistWords * 4;
    }
};

__device__ __forceinline__ int64_t row_of(const Params &p, int b, int64_t pos, bool *ok) {
    if (p.block_table == nullptr) return (int64_t)b * p.seq_stride + pos;
    int64_t page = pos / p.page_size;
    if (page >= p.max_pages) { *ok = false; return 0; }
    int32_t id = __ldg(p.block_table + (int64_t)b * p.max_pages + page);
    int64_t row = (int64_t)id * p.page_size + pos % p.page_size;
    if (id < 0 || row >= p.num_rows) { *ok = false; return 0; }
    return row;
}

// The indexer work of CTA `cta` of `ncta`, by all kThreads threads of the CTA;
// `smem` is the CTA's 1024-byte aligned dynamic shared memory.  On return no
// copy or MMA is in flight, TMEM is released and the mbarriers are
// invalidated, so the caller may reuse the shared memory.
__device__ __forceinline__ void run_indexer(const CUtensorMap *tmap_k_p, const CUtensorMap *tmap_ks_p,
                                            const CUtensorMap *tmap_q_p, const Params &p, uint8_t *smem, int cta,
                                            int ncta) {
    const CUtensorMap &tmap_k = *tmap_k_p, &tmap_ks = *tmap_ks_p, &tmap_q = *tmap_q_p;
    const int S = p.stages, T = p.T, B = p.B, N = 16 * T, GE = p.groups, AB = p.acc_bufs;
    Layout lay(S, T, B, p.hist_rows, p.q_resident != 0);
    Bars *bars = reinterpret_cast<Bars *>(smem + lay.bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.tmem_off);
    int32_t *seq_len = reinterpret_cast<int32_t *>(smem + lay.len_off);     // [B]
    int32_t *tile_pre = reinterpret_cast<int32_t *>(smem + lay.tile_off);   // [B+1] exclusive prefix of tiles

    const int warp = warp_id(), lane = lane_id();

    // --- per-sequence visible lengths (max over its queries) and tile counts
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        int32_t mx = -1;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            int32_t q = __ldg(p.q_pos + b * T + t);
            if (q < 0) ok = false;
            mx = max(mx, q);
        }
        int64_t cap = p.block_table ? (int64_t)p.max_pages * p.page_size : p.seq_stride;
        if (!ok || (int64_t)mx >= cap || (int64_t)mx >= p.Lmax) {
            ok = false;
        }
        if (!ok) {
            if (cta == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
            mx = -1;
        }
        seq_len[b] = mx + 1;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < B; base += 32) {
            int b = base + lane;
            int v = b < B ? (seq_len[b] + kTile - 1) / kTile : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (b < B) tile_pre[b + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) tile_pre[0] = 0;
    }
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + lay.hist_off);   // [hist_rows][2048] or empty
    for (int j = threadIdx.x; j < p.hist_rows * kHistWords; j += blockDim.x) hist[j] = 0;
    __syncthreads();

    const int total = tile_pre[B];
    const int per = total / ncta, rem = total % ncta;
    const int t_begin = cta * per + min(cta, rem);
    const int n_tiles = per + (cta < rem ? 1 : 0);
    if (n_tiles == 0) return;   // uniform across the CTA
    // the CTA's range, split in two contiguous halves, one per pipeline
    const int half = (n_tiles + kPipes - 1) / kPipes;
    auto pipe_begin = [&](int pp) { return t_begin + min(n_tiles, pp * half); };
    auto pipe_count = [&](int pp) { return min(n_tiles, (pp + 1) * half) - min(n_tiles, pp * half); };

    // --- barriers and TMEM (GE accumulators of N columns per pipeline)
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)(kPipes * GE * AB * N)) tmem_cols <<= 1;
    if (threadIdx.x == 0) {
        for (int pp = 0; pp < kPipes; ++pp) {
            for (int s = 0; s < S; ++s) {
                mbar_init(&bars->full[pp][s], 1);
                mbar_init(&bars->empty[pp][s], 1 + kEpiWarps);
            }
            for (int a = 0; a < GE; ++a)
                for (int u = 0; u < AB; ++u) {
                    mbar_init(&bars->tfull[pp][a][u], 1);
                    mbar_init(&bars->tempty[pp][a][u], kEpiWarps);
                }
            mbar_init(&bars->mma_done[pp], 1);
        }
        mbar_init(&bars->q_full, 1);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_ks);
        prefetch_tmap(&tmap_q);
    }
    if (warp == kPipes) {   // the first MMA warp owns the TMEM allocation
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // (sequence, tile) of global tile g
    auto locate = [&](int g, int &b, int &ti) {
        int lo = 0, hi = B - 1;
        while (lo < hi) {   // last b with tile_pre[b] <= g
            int mid = (lo + hi + 1) >> 1;
            if (tile_pre[mid] <= g) lo = mid; else hi = mid - 1;
        }
        b = lo;
        while (b < B - 1 && tile_pre[b + 1] <= g) ++b;   // skip empty sequences
        ti = g - tile_pre[b];
    };
    auto stage_of = [&](int pp, int s) { return pp * S + s; };

    const uint32_t stage_tx = kTile * kKeyBytes + kTile * 4 + (p.q_resident ? 0 : N * kKeyBytes);

    if (warp < kPipes) {
        // ------------------------------------------------------------ producer
        const int pp = warp;
        const int n_p = pipe_count(pp);
        if (lane == 0 && n_p > 0) {
            const uint64_t stream_policy = l2_evict_first_policy();   // keys and scales are read once
            int b, ti;
            locate(pipe_begin(pp), b, ti);
            int issued = 0;
            for (int i = 0; i < n_p; ++i) {
                const int s = i % S, st = stage_of(pp, s);
                if (i >= S && !mbar_wait(&bars->empty[pp][s], ((i / S) & 1) ^ 1, p.status)) break;
                mbar_arrive_expect_tx(&bars->full[pp][s], stage_tx);
                uint8_t *kdst = smem + lay.k_off + st * kTile * kKeyBytes;
                uint8_t *ksdst = smem + lay.ks_off + st * kKsStageBytes;
                if (pp == 0 && i == 0 && p.q_resident) {   // the one query block, once
                    mbar_arrive_expect_tx(&bars->q_full, N * kKeyBytes);
                    tma_load_2d(smem + lay.q_off, &tmap_q, &bars->q_full, 0, 0);
                }
                if (!p.q_resident)
                    tma_load_2d(smem + lay.q_off + st * N * kKeyBytes, &tmap_q, &bars->full[pp][s], 0, b * T * 16);
                const int R = p.rows_per_load;
                for (int j = 0; j < kTile / R; ++j) {
                    int64_t pos = (int64_t)ti * kTile + j * R;
                    bool ok = true;
                    int64_t row = 0;
                    if (pos < seq_len[b]) {
                        row = row_of(p, b, pos, &ok);
                        if (!ok) { flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX); row = 0; }
                    }
                    tma_load_2d_hint(kdst + j * R * kKeyBytes, &tmap_k, &bars->full[pp][s], 0, (int32_t)row,
                                     stream_policy);
                    tma_load_1d_hint(ksdst + ks_slot_offset(j * R, R), &tmap_ks, &bars->full[pp][s], (int32_t)row,
                                     stream_policy);
                }
                ++issued;
                if (++ti * kTile >= seq_len[b]) {   // next non-empty sequence
                    ti = 0;
                    do { ++b; } while (b < B && seq_len[b] == 0);
                }
            }
            // drain: never leave a copy in flight into shared memory
            for (int i = max(0, issued - S); i < issued; ++i)
                mbar_wait(&bars->full[pp][i % S], (i / S) & 1, p.status);
            if (pp == 0 && p.q_resident && issued > 0) mbar_wait(&bars->q_full, 0, p.status);
        }
    } else if (warp < 2 * kPipes) {
        // ---------------------------------------------------------- MMA issuer
        const int pp = warp - kPipes;
        const int n_p = pipe_count(pp);
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3_f32(kTile, N);
            for (int i = 0; i < n_p; ++i) {
                const int s = i % S, st = stage_of(pp, s), a = i % GE;
                const int jj = i / GE, u = jj % AB;   // the group's jj-th tile, its accumulator
                if (!mbar_wait(&bars->full[pp][s], (i / S) & 1, p.status)) break;
                if (jj >= AB && !mbar_wait(&bars->tempty[pp][a][u], ((jj / AB) & 1) ^ 1, p.status)) break;
                if (i == 0 && p.q_resident && !mbar_wait(&bars->q_full, 0, p.status)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + lay.k_off + st * kTile * kKeyBytes);
                const uint32_t b_addr = smem_u32(smem + lay.q_off + (p.q_resident ? 0 : st * N * kKeyBytes));
                const uint32_t d = tmem_base + (uint32_t)(((pp * GE + a) * AB + u) * N);
#pragma unroll
                for (int k = 0; k < kKeyBytes / 32; ++k)
                    umma_f8(d, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                            k > 0 ? 1u : 0u);
                umma_commit(&bars->empty[pp][s]);
                umma_commit(&bars->tfull[pp][a][u]);
            }
            umma_commit(&bars->mma_done[pp]);
            mbar_wait(&bars->mma_done[pp], 0, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;                 // 0 .. kPipes*kMaxGroups*4 - 1
        const int pp = ew / (kMaxGroups * kEpiWarps);    // pipeline
        const int a = (ew / kEpiWarps) % kMaxGroups;     // group == accumulator
        const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
        const int row_in_tile = quarter * 32 + lane;
        const int n_p = pipe_count(pp), g0 = pipe_begin(pp);
        float *coef = reinterpret_cast<float *>(smem + lay.epi_off) + ew * (17 * T);
        int32_t *qp = reinterpret_cast<int32_t *>(coef + 16 * T);
        const uint32_t acc_col0 = (uint32_t)((pp * GE + a) * AB * N);
        int cur_b = -1;
        for (int i = a; i < n_p && a < GE; i += GE) {
            const int s = i % S, st = stage_of(pp, s);
            int b, ti;
            locate(g0 + i, b, ti);
            if (b != cur_b) {   // per-sequence constants: w * q_scale and query positions
                __syncwarp();
                for (int j = lane; j < 16 * T; j += 32)
                    coef[j] = __ldg(p.w + (int64_t)b * 16 * T + j) * __ldg(p.q_scale + (int64_t)b * 16 * T + j);
                for (int j = lane; j < T; j += 32) qp[j] = __ldg(p.q_pos + b * T + j);
                __syncwarp();
                cur_b = b;
            }
            const int jj = i / GE, u = jj % AB;
            const uint32_t acc_col = acc_col0 + (uint32_t)(u * N);
            bool ok = mbar_wait(&bars->tfull[pp][a][u], (jj / AB) & 1, p.status) &&
                      mbar_wait(&bars->full[pp][s], (i / S) & 1, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;   // keep the warp converged for tcgen05.ld
            tc_fence_after();
            const float ks = *reinterpret_cast<const float *>(smem + lay.ks_off + st * kKsStageBytes +
                                                              ks_slot_offset(row_in_tile, p.rows_per_load));
            const int64_t pos = (int64_t)ti * kTile + row_in_tile;
            const int len = seq_len[b];
            float *out = p.scores + (int64_t)b * T * p.scores_stride + pos;
            for (int t = 0; t < T; ++t) {
                float acc[16];
                tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + acc_col + (uint32_t)(16 * t), acc);
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < 16; ++h) sum = fmaf(coef[16 * t + h], fmaxf(acc[h], 0.f), sum);
                const bool visible = pos < len && pos <= qp[t];
                if (pos < len) out[(int64_t)t * p.scores_stride] = visible ? ks * sum : -INFINITY;
                if (p.hist_rows) {   // histogram of the visible scores
                    const uint32_t key = float_order_key(ks * sum);
                    const uint32_t bin = (key >> 31) ? ((key >> 20) & (kHistBins - 1)) : (uint32_t)kHistBins;
                    warp_hist_add(hist, (b * T + t) * kHistWords + bin, visible);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->tempty[pp][a][u]);
                mbar_arrive(&bars->empty[pp][s]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kPipes) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
    if (threadIdx.x == 0) {
        for (int pp = 0; pp < kPipes; ++pp) {
            for (int s = 0; s < S; ++s) {
                mbar_inval(&bars->full[pp][s]);
                mbar_inval(&bars->empty[pp][s]);
            }
            for (int a = 0; a < GE; ++a)
                for (int u = 0; u < AB; ++u) {
                    mbar_inval(&bars->tfull[pp][a][u]);
                    mbar_inval(&bars->tempty[pp][a][u]);
                }
            mbar_inval(&bars->mma_done[pp]);
        }
        mbar_inval(&bars->q_full);
    }
    // add this CTA's histogram into the rows' global histograms
    for (int j = threadIdx.x; j < p.hist_rows * kHistWords; j += blockDim.x)
        if (hist[j]) atomicAdd(p.hist_global + (int64_t)(j / kHistWords) * p.hist_row_words + (j % kHistWords), hist[j]);
    __syncthreads();
}

}  // namespace indexer
}  // namespace dsa

namespace dsa {
// Prepared launch of the indexer body (see prepare_indexer in kernels.h).
struct IndexerLaunch {
    CUtensorMap tmap_k, tmap_ks, tmap_q;
    indexer::Params p;
    size_t smem = 0;
    int grid = 0;
};
}  // namespace dsa
