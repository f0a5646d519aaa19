// indexer.cu -- streaming lightning indexer on the 5th-generation tensor cores.
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
// Design (persistent, two CTAs per SM, warp-specialised):
//   warp 0  TMA producer: per 128-key tile, loads the e4m3 key tile
//           [128 x 128 B] (128-byte swizzle), the 128 fp32 key scales and the
//           query's index heads [16T x 128 B] into one pipeline stage.
//   warp 1  MMA issuer: D[128 keys x 16T] += K_tile[128 x 32] * Q^T[32 x 16T]
//           with tcgen05.mma kind::f8f6f4 (four K=32 steps), fp32 accumulators
//           in TMEM, one accumulator per epilogue group so the epilogue of
//           tile i overlaps the MMA of tile i + 1.
//   warps 2-9 epilogue, two groups of four warps (one per TMEM lane quarter),
//           each group with its own accumulator and every other tile:
//           tcgen05.ld of one key row per thread, ReLU, per-head weighting, key
//           scale, causal mask, coalesced fp32 store.
// Each CTA owns a contiguous range of the (sequence, tile) list, so the HBM
// stream of every SM is sequential.
#pragma once

#include "common.cuh"

namespace dsa {
namespace indexer {

constexpr int kTile = 128;            // keys per tile = UMMA M
constexpr int kKeyBytes = DSA_INDEX_DIM;  // 128 e4m3 codes per key
constexpr int kMaxGroups = 2;         // epilogue groups (4 warps each), one TMEM accumulator per group
constexpr int kThreads = 64 + 128 * kMaxGroups;
// Two CTAs share each SM: a single CTA's TMA pipeline does not reach the
// per-SM share of HBM bandwidth on its own (measured: 0.65 us per 16 KB tile
// with one pipeline per SM, twice the throughput with two).  Each CTA keeps
// its shared memory under half an SM and its TMEM under 256 columns.
constexpr int kCtasPerSm = 2;
constexpr int kMaxTmemCols = 512 / kCtasPerSm;
constexpr int kEpiWarps = 4;          // warps per epilogue group (one per TMEM lane quarter)
constexpr int kKsStageBytes = 1024;   // key-scale slots of one stage
constexpr int kHistBins = 2048;       // first radix digit of the selection (11 bits)

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
    int stages;
    int rows_per_load;   // R: rows per TMA box (128, or the page size when pages are smaller)
    int groups;          // epilogue groups in use (1..kMaxGroups)
    // optional first-digit histogram of the visible scores (top 11 bits of
    // the order key), added into hist_global[row * hist_row_words + bin] for
    // rows b * T + t < hist_rows; hist_rows == 0 turns it off
    int hist_rows;
    int hist_row_words;
    uint32_t *hist_global;
};

struct __align__(8) Bars {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t tfull[kMaxGroups];
    uint64_t tempty[kMaxGroups];
    uint64_t mma_done;
};

// Shared memory carve-up (base aligned to 1024 bytes):
//   [0, S*16K)                    key tiles
//   [S*16K, S*(16K + 2K*T))       query tiles
//   then S*1 KB                   key scales: one 128-byte aligned slot per TMA
//                                 box (tensor copies need 128-byte aligned
//                                 shared destinations), R*4 bytes used per slot
//   then Bars, tmem address, per-sequence tables, per-warp epilogue constants,
//   optional per-row score histograms
struct Layout {
    uint32_t k_off, q_off, ks_off, bar_off, tmem_off, len_off, tile_off, epi_off, hist_off, total;
    __host__ __device__ Layout(int S, int T, int B, int hist_rows = 0) {
        k_off = 0;
        q_off = k_off + S * kTile * kKeyBytes;
        ks_off = q_off + S * 16 * T * kKeyBytes;
        bar_off = ks_off + S * kKsStageBytes;
        tmem_off = bar_off + (uint32_t)sizeof(Bars);
        len_off = (tmem_off + 16 + 15) & ~15u;
        tile_off = len_off + 4 * (B + 1);
        tile_off = (tile_off + 15) & ~15u;
        epi_off = tile_off + 4 * (B + 1);
        epi_off = (epi_off + 15) & ~15u;
        // per epilogue warp: 16*T coefficients + T positions
        hist_off = epi_off + kMaxGroups * kEpiWarps * (16 * T + T) * 4;
        total = hist_off + hist_rows * kHistBins * 4;
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
    const int S = p.stages, T = p.T, B = p.B, N = 16 * T;
    Layout lay(S, T, B, p.hist_rows);
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
    for (int j = threadIdx.x; j < p.hist_rows * kHistBins; j += blockDim.x) hist[j] = 0;
    __syncthreads();

    const int total = tile_pre[B];
    const int per = total / ncta, rem = total % ncta;
    const int t_begin = cta * per + min(cta, rem);
    const int n_tiles = per + (cta < rem ? 1 : 0);
    if (n_tiles == 0) return;   // uniform across the CTA

    // --- barriers and TMEM (one N-column fp32 accumulator per epilogue group)
    const int GE = p.groups;
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)(GE * N)) tmem_cols <<= 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1 + kEpiWarps);
        }
        for (int a = 0; a < GE; ++a) {
            mbar_init(&bars->tfull[a], 1);
            mbar_init(&bars->tempty[a], kEpiWarps);
        }
        mbar_init(&bars->mma_done, 1);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_ks);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // cursor over the (sequence, tile) list starting at global tile t_begin
    auto locate = [&](int g, int &b, int &ti) {
        int lo = 0, hi = B - 1;
        while (lo < hi) {   // last b with tile_pre[b] <= g and a non-empty range
            int mid = (lo + hi + 1) >> 1;
            if (tile_pre[mid] <= g) lo = mid; else hi = mid - 1;
        }
        b = lo;
        while (b < B - 1 && tile_pre[b + 1] <= g) ++b;   // skip empty sequences
        ti = g - tile_pre[b];
    };

    const uint32_t stage_tx = kTile * kKeyBytes + kTile * 4 + N * kKeyBytes;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int b, ti;
            locate(t_begin, b, ti);
            int issued = 0;
            bool alive = true;
            for (int i = 0; i < n_tiles && alive; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(&bars->empty[s], ((i / S) & 1) ^ 1, p.status)) { alive = false; break; }
                mbar_arrive_expect_tx(&bars->full[s], stage_tx);
                uint8_t *kdst = smem + lay.k_off + s * kTile * kKeyBytes;
                uint8_t *ksdst = smem + lay.ks_off + s * kKsStageBytes;
                tma_load_2d(smem + lay.q_off + s * N * kKeyBytes, &tmap_q, &bars->full[s], 0, b * T * 16);
                const int R = p.rows_per_load;
                for (int j = 0; j < kTile / R; ++j) {
                    int64_t pos = (int64_t)ti * kTile + j * R;
                    bool ok = true;
                    int64_t row = 0;
                    if (pos < seq_len[b]) {
                        row = row_of(p, b, pos, &ok);
                        if (!ok) { flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX); row = 0; }
                    }
                    tma_load_2d(kdst + j * R * kKeyBytes, &tmap_k, &bars->full[s], 0, (int32_t)row);
                    tma_load_1d(ksdst + ks_slot_offset(j * R, R), &tmap_ks, &bars->full[s], (int32_t)row);
                }
                ++issued;
                if (++ti * kTile >= seq_len[b]) {   // next non-empty sequence
                    ti = 0;
                    do { ++b; } while (b < B && seq_len[b] == 0);
                }
            }
            // drain: never leave a copy in flight into shared memory
            for (int i = max(0, issued - S); i < issued; ++i)
                mbar_wait(&bars->full[i % S], (i / S) & 1, p.status);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3_f32(kTile, N);
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i % S, a = i % GE;
                if (!mbar_wait(&bars->full[s], (i / S) & 1, p.status)) break;
                if (i >= GE && !mbar_wait(&bars->tempty[a], ((i / GE) & 1) ^ 1, p.status)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + lay.k_off + s * kTile * kKeyBytes);
                const uint32_t b_addr = smem_u32(smem + lay.q_off + s * N * kKeyBytes);
                const uint32_t d = tmem_base + (uint32_t)(a * N);
#pragma unroll
                for (int k = 0; k < kKeyBytes / 32; ++k)
                    umma_f8(d, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                            k > 0 ? 1u : 0u);
                umma_commit(&bars->empty[s]);
                umma_commit(&bars->tfull[a]);
            }
            umma_commit(&bars->mma_done);
            mbar_wait(&bars->mma_done, 0, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // group e (warps 2+4e .. 5+4e) takes tiles e, e + GE, e + 2 GE, ... into accumulator e
        const int ew = warp - 2;                  // 0..15
        const int a = ew / kEpiWarps;             // group == accumulator
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int row_in_tile = quarter * 32 + lane;
        float *coef = reinterpret_cast<float *>(smem + lay.epi_off) + ew * (17 * T);
        int32_t *qp = reinterpret_cast<int32_t *>(coef + 16 * T);
        int cur_b = -1;
        for (int i = a; i < n_tiles && a < GE; i += GE) {
            const int s = i % S;
            int b, ti;
            locate(t_begin + i, b, ti);
            if (b != cur_b) {   // per-sequence constants: w * q_scale and query positions
                __syncwarp();
                for (int j = lane; j < 16 * T; j += 32)
                    coef[j] = __ldg(p.w + (int64_t)b * 16 * T + j) * __ldg(p.q_scale + (int64_t)b * 16 * T + j);
                for (int j = lane; j < T; j += 32) qp[j] = __ldg(p.q_pos + b * T + j);
                __syncwarp();
                cur_b = b;
            }
            bool ok = mbar_wait(&bars->tfull[a], (i / GE) & 1, p.status) &&
                      mbar_wait(&bars->full[s], (i / S) & 1, p.status);
            if (!__all_sync(0xffffffffu, ok)) break;   // keep the warp converged for tcgen05.ld
            tc_fence_after();
            const float ks = *reinterpret_cast<const float *>(smem + lay.ks_off + s * kKsStageBytes +
                                                              ks_slot_offset(row_in_tile, p.rows_per_load));
            const int64_t pos = (int64_t)ti * kTile + row_in_tile;
            const int len = seq_len[b];
            float *out = p.scores + (int64_t)b * T * p.scores_stride + pos;
            for (int t = 0; t < T; ++t) {
                float acc[16];
                tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * N + 16 * t), acc);
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < 16; ++h) sum = fmaf(coef[16 * t + h], fmaxf(acc[h], 0.f), sum);
                const bool visible = pos < len && pos <= qp[t];
                if (pos < len) out[(int64_t)t * p.scores_stride] = visible ? ks * sum : -INFINITY;
                if (p.hist_rows) {   // first-digit histogram of the visible scores (warp-aggregated)
                    const uint32_t bin = visible ? (b * T + t) * kHistBins + (float_order_key(ks * sum) >> 21)
                                                 : 0xFFFFFFFFu;
                    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                    if (visible && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->tempty[a]);
                mbar_arrive(&bars->empty[s]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_inval(&bars->full[s]);
            mbar_inval(&bars->empty[s]);
        }
        for (int a = 0; a < GE; ++a) {
            mbar_inval(&bars->tfull[a]);
            mbar_inval(&bars->tempty[a]);
        }
        mbar_inval(&bars->mma_done);
    }
    // add this CTA's histogram into the rows' global histograms
    for (int j = threadIdx.x; j < p.hist_rows * kHistBins; j += blockDim.x)
        if (hist[j]) atomicAdd(p.hist_global + (int64_t)(j / kHistBins) * p.hist_row_words + (j % kHistBins), hist[j]);
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
