// capture.cu -- the DSA decode layer-step for up to four long query rows as
// one cooperative kernel with a single grid barrier after the key stream.
//
// What it computes is exactly the layer-step of dsa_layer_decode: indexer
// scores of every visible key, the top-k positions with ties to the lower
// position, sparse GQA attention over them with the sink ("Naive-N0.5-Flash:
// no full-attention layers, and a runtime built by AI", sections "Inside a DSA
// layer: the lightning indexer" and "What 'no full-attention layers' means").
// How it is organised is this library's own design for B200: the selection
// work that depends on every score is cut down to a short list that the key
// stream itself produces.
//
// Phase 1, the key stream (one CTA per SM, two TMA -> tcgen05 pipelines with
// two TMEM accumulators per epilogue group, four epilogue groups of four
// warps; indexer_impl.cuh has the machinery).  The epilogue scores and
// stores as the standalone indexer does; besides, each group's first tile is
// a sample: its 8-bins-per-octave histogram goes into the CTA's shared
// histogram, the CTA's last group adds it into the row's global one, and the
// last CTA to do so turns each row's histogram into a score threshold -- a
// bin edge below which the sample predicts about `oversample` x top_k keys --
// and publishes it.  The thresholds arrive in the middle of the stream: one
// warp per epilogue group polls for them between tiles, and from then on each
// epilogue warp keeps, tile by tile, every visible key of its 32 rows at or
// above its row's threshold in a short list of its own in shared memory (the
// tiles it scored before, it takes again from its own stored scores).  When
// its tiles are done, a CTA merges its warps' lists into its segment of the
// row's candidate list, in position order.
// One grid barrier.  The segments' lengths tell whether the sample was good:
// if every row holds at least top_k candidates (then the list holds every key
// at or above the k-th largest score, since the threshold is below it) and no
// segment overflowed, the fast path runs; otherwise the general path of the
// fused layer-step does (the result is the same either way).
// Phase 2 (fast), per CTA of a row that has attention units: the row's
// candidates (a few thousand) into shared memory in position order (one bulk
// copy per segment), the exact k-th largest key (one wide histogram of the
// bits below the keys' common ones, then the few keys of its bin), the
// selection compacted in position order into shared memory.  Each team of the
// CTA then runs a 64-key attention unit from there, and once every unit of
// its (row, KV group) has written its partial, combines one slice of that
// group's outputs with the sink, with the combine kernel's arithmetic.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "attention_impl.cuh"
#include "indexer_impl.cuh"
#include "kernels.h"
#include "topk_impl.cuh"

namespace dsa {
namespace capture {

using indexer::kEpiWarp0;
using indexer::kEpiWarps;
using indexer::kKeyBytes;
using indexer::kMaxGroups;
using indexer::kPipes;
using indexer::kTile;

constexpr int kThreads = indexer::kThreads;   // 640
constexpr int kWarps = kThreads / 32;
constexpr int kTeams = 4;                     // attention teams of 4 warps (named barriers 1..4)
constexpr int kMaxRows = 4;                   // B * T on this path
constexpr int kGroups = kPipes * kMaxGroups;  // epilogue groups per CTA
constexpr int kBins = 2048;                   // sample histogram: bits 30..20 of the non-negative keys
constexpr int kHistWords = kBins + 1;         // + the count of negative scores
constexpr int kHistStride = kHistWords + 3;   // words between rows' histograms: rows start 16-byte aligned
constexpr int kSegCap = 1024;                 // candidates one CTA may hold per row
constexpr int kWarpCap = 64;                  // candidates one epilogue warp may hold per row
constexpr int kMaxBacklog = 16;               // tiles per epilogue group whose keys wait in TMEM for the thresholds
constexpr int kListCap = 16384;               // candidates of one row the selection takes into shared memory
constexpr int kWide = 4096;                   // bins of the selection's first histogram
constexpr int kSmall = 2048;                  // keys of T*'s bin taken aside for the remaining bits
// The candidates' histogram that the stream builds: bin (key - threshold) >>
// kCandShift, kWide bins, the last one taking everything above (two octaves
// of non-negative scores at 1/2048 octave).
constexpr int kCandShift = 12;
constexpr int kGroupBar0 = 5;                 // named barriers 5..8: the epilogue groups
constexpr int kUnitBar = 9;                   // named barrier of the attention teams of a CTA unit
constexpr int kSelBytes = DSA_MAX_TOPK * 4;   // the selection, at the start of shared memory in phase 2
constexpr int64_t kMinContext = 8192;         // shorter contexts take the fused layer-step
// attention units per (row, KV head) for top_k <= DSA_MAX_TOPK
constexpr int kMaxSplits = (DSA_MAX_TOPK + kAttnChunk - 1) / kAttnChunk;

// control words at the start of the capture scratch
enum {
    kGridArrive = 0,
    kGridExit = 1,
    kSampleArrive = 2,
    kReady = 3,
    kOverflow = 4,
    kThr = 8,                 // [kMaxRows] thresholds (order keys)
    kTotal = 12,              // [kMaxRows] candidates per row
    kCombine = 16,            // [kMaxRows][64] attention units done per (row, KV group)
    kThrPacked = 272,         // [kMaxRows] 64-bit: (1 << 32) | threshold, once published
    kCtlWords = 512
};

static_assert(kCombine + kMaxRows * DSA_Q_HEADS <= kThrPacked && kThrPacked + 2 * kMaxRows <= kCtlWords,
              "control words");
static_assert(kThrPacked % 2 == 0, "64-bit words");
static_assert(kTeams * 4 < kWarps, "the attention teams must leave warps free in the CTA");

struct Params {
    indexer::Params ix;
    topk::Params tk;          // the general selection (fallback)
    attn::Params at;
    const float *sink;
    __nv_bfloat16 *O;
    float *lse;
    uint32_t *ctl;
    uint32_t *sample_hist;    // [rows][kHistStride]
    uint32_t *counts;         // [rows][NG]
    uint32_t *cand_hist;      // [rows][kWide] the candidates' keys above the row's threshold (kCandShift)
    uint2 *lists;             // [rows][NG][kSegCap] (order key, position)
    uint32_t *path_count;     // [2] calls that took the fast path / the general path
    uint64_t *trace;          // [grid][DSA_TRACE_MARKS] phase marks, or NULL
    const float *k_scale;     // the index keys' scales, [cache rows]
    BarrierCfg bar;
    int rows, K, C, NG;
    float oversample;
};

__host__ __device__ constexpr size_t align128(size_t x) { return (x + 127) & ~size_t(127); }

// Shared memory of phase 1 (base aligned to 1024 bytes).
struct Layout {
    uint32_t k_off, q_off, ks_off, bar_off, tmem_off, len_off, tile_off, epi_off, hist_off, misc_off, cap_off, poll_off,
        total;
    __host__ __device__ Layout(int S, int T, int B) {
        const int stages = kPipes * S, rows = B * T;
        k_off = 0;
        q_off = stages * kTile * kKeyBytes;
        ks_off = q_off + rows * 16 * kKeyBytes;   // every row's query block, resident
        bar_off = ks_off + stages * indexer::kKsStageBytes;
        tmem_off = bar_off + (uint32_t)sizeof(indexer::Bars);
        len_off = (tmem_off + 16 + 15) & ~15u;
        tile_off = (len_off + 4 * (B + 1) + 15) & ~15u;
        epi_off = (tile_off + 4 * (B + 1) + 15) & ~15u;
        hist_off = epi_off + kGroups * kEpiWarps * (16 * T + T) * 4;
        misc_off = hist_off + rows * kHistStride * 4;
        // misc: [0] groups sampled, [1 + g] group g's role in the sample
        // exchange, [5] rows' thresholds published; then the rows' query
        // positions
        // [kMaxRows] thresholds, [kMaxRows] their flag; then per group: the
        // warps' counts of a capture step, the lists' lengths, the decisions
        cap_off = misc_off + 32 + 16;
        poll_off = cap_off + 4 * (2 * kMaxRows + kGroups * (kEpiWarps * kMaxRows + 2 * kMaxRows + 2));
        total = poll_off + kGroups * kMaxRows * 8;   // [group] the packed words, as the poller read them
    }
};

// Bin of a non-negative order key in the sample histogram; kBins for a
// negative score.
__device__ __forceinline__ uint32_t sample_bin(uint32_t key) {
    return (key >> 31) ? ((key >> 20) & (kBins - 1)) : (uint32_t)kBins;
}

// The threshold of one row from its sample histogram (every CTA's sample
// added in), already copied into shared memory `local` (kHistWords words),
// by one warp.
// The sample's visible keys (the histogram's total, tot) predict
// oversample * K * tot / n + 16 of them at or above the row's threshold; the
// threshold lies in the highest bin b whose count, with the bins above it,
// reaches that target, where the part of b's count still needed would lie
// above it were b's keys spread evenly over its key values; zero (take every
// key) when the sample's non-negative scores do not reach the target.  Any
// threshold gives the exact result (a short list takes the general path);
// this one keeps the list near oversample x top_k.
__device__ uint32_t row_threshold(const uint32_t *local, int64_t n, int K, float oversample) {
    const int lane = lane_id();
    constexpr int kPer = kBins / 32;   // 64 bins per lane
    uint32_t s = 0;
    const uint4 *l4 = reinterpret_cast<const uint4 *>(local + lane * kPer);
#pragma unroll
    for (int u = 0; u < kPer / 4; ++u) {
        const uint4 v = l4[u];
        s += v.x + v.y + v.z + v.w;
    }
    const uint32_t negative = local[kBins];
    uint32_t incl = s;   // keys in this lane's bins and all higher ones
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += u;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 0) + negative;
    const double want = (double)oversample * K * (double)tot / (double)n + 16.0;
    const uint32_t target = (uint32_t)min((double)tot, ceil(want));
    const uint32_t hit = __ballot_sync(0xffffffffu, incl >= target);
    uint32_t thr = 0;
    if (target > 0 && hit) {
        const int L = 31 - __clz(hit);   // highest lane whose suffix reaches the target
        const uint32_t above = __shfl_sync(0xffffffffu, incl - s, L);
        // that lane's 64 bins, two per lane, then the same search over them
        const uint32_t b0 = (uint32_t)(L * kPer + 2 * lane);
        const uint32_t v0 = local[b0], v1 = local[b0 + 1];
        const uint32_t t = v0 + v1;
        uint32_t inc2 = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_down_sync(0xffffffffu, inc2, o);
            if (lane + o < 32) inc2 += u;
        }
        // bins b0 + 1 and b0 in descending order
        const uint32_t run1 = above + inc2 - t + v1;   // keys in bins >= b0 + 1
        const uint32_t run0 = run1 + v0;               // keys in bins >= b0
        uint32_t mine = 0xFFFFFFFFu, m_above = 0, m_cnt = 0;
        if (run1 >= target) {
            mine = b0 + 1;
            m_above = run1 - v1;
            m_cnt = v1;
        } else if (run0 >= target) {
            mine = b0;
            m_above = run0 - v0;
            m_cnt = v0;
        }
        const uint32_t best = __reduce_max_sync(0xffffffffu, mine == 0xFFFFFFFFu ? 0u : mine + 1);
        if (best) {
            // inside bin best - 1: the keys above the bins over it fall short
            // of the target by `need` (1 .. its count cb); the threshold is
            // put where `need` of its cb keys would lie above it if they were
            // spread evenly over the bin's 2^20 key values
            const int owner = __ffs(__ballot_sync(0xffffffffu, mine + 1u == best)) - 1;
            const uint32_t ab = __shfl_sync(0xffffffffu, m_above, owner);
            const uint32_t cb = __shfl_sync(0xffffffffu, m_cnt, owner);
            const uint32_t need = target - ab;
            thr = (0x80000000u | ((best - 1) << 20)) + (uint32_t)(((uint64_t)(cb - need) << 20) / cb);
        }
    }
    return thr;
}

// Phase 1: the indexer over this CTA's tiles with sampling and candidate
// capture (see the file comment).  All kThreads threads call it.  On return
// nothing is in flight, TMEM is released and the mbarriers are invalidated;
// keep[0 .. kMaxRows) holds the rows' thresholds if keep[kMaxRows] != 0.
template <int TQ, class AfterWait>
__device__ void run_indexer_capture(const CUtensorMap *tmap_k_p, const CUtensorMap *tmap_ks_p,
                                    const CUtensorMap *tmap_q_p, const Params &cp, uint8_t *smem, int cta, int ncta,
                                    uint32_t *keep, AfterWait &&after_wait) {
    using namespace indexer;
    const indexer::Params &p = cp.ix;
    const CUtensorMap &tmap_k = *tmap_k_p, &tmap_q = *tmap_q_p;
    (void)tmap_ks_p;   // (the key scales are read from global memory by the epilogue)
    // the query tokens per sequence are a compile-time constant: the per-query
    // loops of the epilogue keep only the copies that run (a smaller loop body
    // that stays in the instruction cache)
    constexpr int T = TQ;
    const int S = p.stages, B = p.B, N = 16 * T, GE = p.groups, AB = p.acc_bufs, rows = B * T;
    Layout lay(S, T, B);
    Bars *bars = reinterpret_cast<Bars *>(smem + lay.bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.tmem_off);
    int32_t *seq_len = reinterpret_cast<int32_t *>(smem + lay.len_off);
    int32_t *tile_pre = reinterpret_cast<int32_t *>(smem + lay.tile_off);
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + lay.hist_off);   // [rows][kHistStride]
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + lay.misc_off);   // [0] groups sampled, [1..4] group flags,
                                                                          // [5] rows' thresholds published
    int32_t *row_qpos = reinterpret_cast<int32_t *>(smem + lay.misc_off + 32);   // [rows] query positions
    uint32_t *thr_s = reinterpret_cast<uint32_t *>(smem + lay.cap_off);   // [kMaxRows] thresholds, then the flag
    uint32_t *wcs = thr_s + 2 * kMaxRows;              // [epilogue warp][kMaxRows] the warps' list lengths
    constexpr int kCapWords = 2 * kMaxRows + kGroups * kEpiWarps * kMaxRows;
    // After the sample the histogram area holds the epilogue warps' candidate
    // lists: row r's at hist + r * kHistStride, epilogue warp w's at
    // + w * kWarpCap entries (order key, position), each in position order.
    auto wlist = [&](int r, int w) { return reinterpret_cast<uint2 *>(hist + r * kHistStride) + w * kWarpCap; };
    static_assert(kGroups * kEpiWarps * kWarpCap * 8 <= kHistStride * 4, "warp lists in the histogram area");
    static_assert(kGroups * kEpiWarps * kWarpCap <= kSegCap, "a CTA's warp lists fit its segment");
    uint32_t *ctl = cp.ctl;
    const int warp = warp_id(), lane = lane_id();
    const uint32_t lt = (1u << lane) - 1u;

    // The prologue has one block barrier: thread 0 builds the mbarriers while
    // warp kPipes allocates TMEM and the other threads clear the shared words;
    // then (after the dependent-launch wait) thread 0 reads the (at most
    // kMaxRows) query positions, all loads in flight together, and builds the
    // per-sequence tables.
    // TMEM: the accumulators, then the backlog: the order keys of the first
    // back_cap tiles of each epilogue group, kept until the thresholds come
    // (column acc_cols + (group * back_cap + tile) * T + query, lane = key row)
    const int acc_cols = kPipes * GE * AB * N;
    const int back_cap = min(kMaxBacklog, (512 - acc_cols) / (kGroups * T));
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)(acc_cols + kGroups * back_cap * T)) tmem_cols <<= 1;
    if (threadIdx.x == 0) {
        for (int pp = 0; pp < kPipes; ++pp) {
            for (int s = 0; s < S; ++s) {
                mbar_init(&bars->full[pp][s], 1);
                mbar_init(&bars->empty[pp][s], 1);   // the MMA's commit: the epilogue never reads the stage
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
        prefetch_tmap(&tmap_q);
    }
    if (warp == kPipes) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    for (int j = threadIdx.x; j < rows * kHistStride; j += blockDim.x) hist[j] = 0;
    if (threadIdx.x < 8) misc[threadIdx.x] = 0;
    for (int j = threadIdx.x; j < kCapWords; j += blockDim.x) thr_s[j] = 0;
    // One sequence in a contiguous cache: the first two tiles each pipeline
    // streams when the query sits at the last position the cache holds (a
    // decode step), on their way into L2 -- a guess from the sizes alone, so
    // it reads nothing the previous grid may be writing; a wrong guess only
    // costs the prefetch.
    if (B == 1 && p.block_table == nullptr && warp < kPipes && lane == 0) {
        const int total_g = (int)((p.Lmax + kTile - 1) / kTile);
        const int per_g = total_g / ncta, rem_g = total_g % ncta;
        const int n_g = per_g + (cta < rem_g ? 1 : 0), half_g = (n_g + kPipes - 1) / kPipes;
        const int first = cta * per_g + min(cta, rem_g) + min(n_g, warp * half_g);
        const int cnt = min(n_g, (warp + 1) * half_g) - min(n_g, warp * half_g);
        for (int i = 0; i < min(cnt, 2); ++i) tma_prefetch_2d(&tmap_k, 0, (first + i) * kTile);
    }
    // Everything above touches only this CTA's shared memory and TMEM (and
    // the prefetch): under a programmatic dependent launch it overlaps the
    // previous grid's tail. From here on the kernel reads what that grid may
    // have written.
    pdl_wait();
    after_wait();
    if (threadIdx.x == 0) {
        int32_t qv[kMaxRows];
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) qv[r] = r < rows ? __ldg(p.q_pos + r) : 0;
        const int64_t cap = p.block_table ? (int64_t)p.max_pages * p.page_size : p.seq_stride;
        int pre = 0;
        tile_pre[0] = 0;
#pragma unroll
        for (int b = 0; b < kMaxRows / T; ++b) {   // (B * T <= kMaxRows)
            if (b < B) {
                int32_t mx = -1;
                bool ok = true;
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const int32_t q = qv[b * T + t];
                    if (q < 0) ok = false;
                    mx = max(mx, q);
                }
                if (!ok || (int64_t)mx >= cap || (int64_t)mx >= p.Lmax) {
                    if (cta == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
                    mx = -1;
                }
                seq_len[b] = mx + 1;
                pre += (mx + 1 + kTile - 1) / kTile;
                tile_pre[b + 1] = pre;
            }
        }
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
            if (r < rows) row_qpos[r] = qv[r];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = tile_pre[B];
    const int per = total / ncta, rem = total % ncta;
    const int t_begin = cta * per + min(cta, rem);
    const int n_tiles = per + (cta < rem ? 1 : 0);
    const int half = (n_tiles + kPipes - 1) / kPipes;
    auto pipe_begin = [&](int pp) { return t_begin + min(n_tiles, pp * half); };
    auto pipe_count = [&](int pp) { return min(n_tiles, (pp + 1) * half) - min(n_tiles, pp * half); };
    // the pipe's tiles in order, its i-th tile to group i % GE (one
    // sequential stream per pipeline)
    auto group_count = [&](int pp, int a) { const int c = pipe_count(pp); return c / GE + (a < c % GE ? 1 : 0); };
    auto tile_of = [&](int pp, int i) { return pipe_begin(pp) + i; };

    auto locate = [&](int g, int &b, int &ti) {
        int lo = 0, hi = B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_pre[mid] <= g) lo = mid; else hi = mid - 1;
        }
        b = lo;
        while (b < B - 1 && tile_pre[b + 1] <= g) ++b;
        ti = g - tile_pre[b];
    };
    const uint32_t stage_tx = kTile * kKeyBytes;   // (the key scales go to the epilogue from global memory)
    const bool any_tiles = pipe_count(0) + pipe_count(1) > 0;

    // ---- candidates, by each epilogue warp on its own: warp w of group g
    //      (rows 32 q .. 32 q + 31 of each of the group's tiles, q = w & 3)
    //      keeps the visible keys of its rows at or above their row's
    //      threshold in a list of its own, in the order it scores its tiles --
    //      position order, since a group's tiles come in increasing
    //      position.  No barrier between warps; after the stream the CTA
    //      merges its warps' lists into its segment in position order.
    const int ew_c = warp - kEpiWarp0;   // negative for the other warps
    const int e_gi = ew_c >= 0 ? ew_c / kEpiWarps : 0;
    const int e_pp = e_gi / kMaxGroups, e_a = e_gi % kMaxGroups;
    const int e_q = warp & 3;
    const int e_row = e_q * 32 + lane;   // the lane's row in each tile
    const int e_ng = ew_c >= 0 && e_a < GE ? group_count(e_pp, e_a) : 0;
    bool capturing = false;   // the warp has the thresholds and takes its candidates
    uint32_t thr[kMaxRows] = {0u, 0u, 0u, 0u};   // the rows' thresholds, once known
    uint32_t wc[kMaxRows] = {0u, 0u, 0u, 0u};    // the warp's list lengths (the same in every lane)
    // Of the warp's rows of one tile of sequence b at position pos (one per
    // lane), those with bit t of cand go with key[t] to the end of the warp's
    // list of row b * T + t.
    auto warp_take = [&](int b, uint32_t cand, const uint32_t (&key)[kMaxRows], uint32_t pos) {
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const uint32_t bits = __ballot_sync(0xffffffffu, (cand >> t) & 1u);
            if (bits == 0u) continue;
            const int r = b * T + t;
            uint32_t n = 0u, th = 0u;
#pragma unroll
            for (int rr = 0; rr < kMaxRows; ++rr)
                if (rr == r) {
                    n = wc[rr];
                    th = thr[rr];
                }
            if ((cand >> t) & 1u) {
                const uint32_t slot = n + __popc(bits & lt);
                if (slot < (uint32_t)kWarpCap) wlist(r, ew_c)[slot] = make_uint2(key[t], pos);
                const uint32_t bin = min((key[t] - th) >> kCandShift, (uint32_t)(kWide - 1));
                atomicAdd(cp.cand_hist + (int64_t)r * kWide + bin, 1u);
            }
#pragma unroll
            for (int rr = 0; rr < kMaxRows; ++rr)
                if (rr == r) wc[rr] += __popc(bits);
        }
    };
    // The warp's backlog: the group's tiles [0, j_now), scored before the
    // thresholds were known; the first back_cap of them from TMEM, the rest
    // from the scores this lane stored (a lane reads back only its own
    // stores), a few tiles' loads in flight at a time.
    auto transition = [&](int j_now) {
        capturing = true;
        __threadfence_block();   // the thresholds, after the flag that announced them
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) thr[r] = r < rows ? thr_s[r] : 0u;
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");   // the backlog's keys are in TMEM
        const int nb = min(j_now, back_cap);
        for (int jj = 0; jj < nb; ++jj) {
            int bb, ti;
            locate(tile_of(e_pp, jj * GE + e_a), bb, ti);
            const int ps = ti * kTile + e_row;
            uint32_t key[kMaxRows] = {0u, 0u, 0u, 0u}, cand = 0u;
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const int r = bb * T + t;
                key[t] = tmem_ld1(tmem_base + ((uint32_t)(e_q * 32) << 16) +
                                  (uint32_t)(acc_cols + (e_gi * back_cap + jj) * T + t));
                if (ps < seq_len[bb] && ps <= row_qpos[r] && key[t] >= thr_s[r]) cand |= 1u << t;
            }
            warp_take(bb, cand, key, (uint32_t)ps);
        }
        constexpr int kB = T <= 2 ? 4 : 2;
        for (int jb = nb; jb < j_now; jb += kB) {
            float v[kB][T];
            int32_t ps[kB];   // (positions below 2^31)
            int bb[kB];
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                bb[u] = 0;
                ps[u] = -1;
                if (jb + u < j_now) {
                    int ti;
                    locate(tile_of(e_pp, (jb + u) * GE + e_a), bb[u], ti);
                    ps[u] = ti * kTile + e_row;
                    if (ps[u] >= seq_len[bb[u]]) ps[u] = -1;
                }
#pragma unroll
                for (int t = 0; t < T; ++t)
                    v[u][t] = ps[u] >= 0 ? p.scores[((int64_t)bb[u] * T + t) * p.scores_stride + ps[u]] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                if (jb + u < j_now) {   // uniform in the warp
                    uint32_t key[kMaxRows] = {0u, 0u, 0u, 0u}, cand = 0u;
#pragma unroll
                    for (int t = 0; t < T; ++t) {
                        const int r = bb[u] * T + t;
                        key[t] = float_order_key(v[u][t]);
                        if (ps[u] >= 0 && ps[u] <= row_qpos[r] && key[t] >= thr_s[r]) cand |= 1u << t;
                    }
                    warp_take(bb[u], cand, key, (uint32_t)ps[u]);
                }
            }
        }
    };
    // the thresholds from their packed words (all rows published), into
    // shared memory for the CTA's warps
    const uint64_t *packed = reinterpret_cast<const uint64_t *>(ctl + kThrPacked);
    auto all_published = [&](const uint64_t (&w)[kMaxRows]) {
        bool ok = true;
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
            if (r < rows) ok &= (w[r] >> 32) != 0u;
        return ok;
    };
    auto wait_packed = [&](uint64_t (&w)[kMaxRows]) {   // bounded
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
#pragma unroll
            for (int r = 0; r < kMaxRows; ++r) w[r] = r < rows ? ld_relaxed_gpu_u64(packed + r) : 0ull;
            if (all_published(w)) return true;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                flag_timeout(p.status);
                return false;
            }
            __nanosleep(64);
        }
    };
    auto publish = [&](const uint64_t (&w)[kMaxRows]) {
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
            if (r < rows) thr_s[r] = (uint32_t)w[r];
        __threadfence_block();
        *reinterpret_cast<volatile uint32_t *>(thr_s + kMaxRows) = 1u;
        if (cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 1] = globaltimer_ns();
    };

    if (warp < kPipes) {
        // ------------------------------------------------------------ producer
        const int pp = warp;
        const int n_p = pipe_count(pp);
        if (lane == 0 && n_p > 0) {
            const uint64_t stream_policy = l2_evict_first_policy();
            int issued = 0;
            for (int i = 0; i < n_p; ++i) {
                const int s = i % S, st = pp * S + s;
                if (i >= S && !mbar_wait(&bars->empty[pp][s], ((i / S) & 1) ^ 1, p.status)) break;
                if (pp == 0 && i == 0) {   // every row's query block, once
                    mbar_arrive_expect_tx(&bars->q_full, rows * 16 * kKeyBytes);
                    for (int b = 0; b < B; ++b)
                        tma_load_2d(smem + lay.q_off + b * N * kKeyBytes, &tmap_q, &bars->q_full, 0, b * N);
                }
                if (i == 0 && pp == 0 && cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 10] = globaltimer_ns();
                mbar_arrive_expect_tx(&bars->full[pp][s], stage_tx);
                int b, ti;
                locate(tile_of(pp, i), b, ti);
                uint8_t *kdst = smem + lay.k_off + st * kTile * kKeyBytes;
                const int R = p.rows_per_load;
                for (int j = 0; j < kTile / R; ++j) {
                    const int64_t pos = (int64_t)ti * kTile + j * R;
                    bool ok = true;
                    int64_t row = 0;
                    if (pos < seq_len[b]) {
                        row = row_of(p, b, pos, &ok);
                        if (!ok) { flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX); row = 0; }
                    }
                    tma_load_2d_hint(kdst + j * R * kKeyBytes, &tmap_k, &bars->full[pp][s], 0, (int32_t)row,
                                     stream_policy);
                }
                ++issued;
            }
            for (int i = max(0, issued - S); i < issued; ++i)
                mbar_wait(&bars->full[pp][i % S], (i / S) & 1, p.status);
            if (pp == 0 && issued > 0) mbar_wait(&bars->q_full, 0, p.status);
        }
    } else if (warp < 2 * kPipes) {
        // ---------------------------------------------------------- MMA issuer
        const int pp = warp - kPipes;
        const int n_p = pipe_count(pp);
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3_f32(kTile, N);
            for (int i = 0; i < n_p; ++i) {
                const int s = i % S, st = pp * S + s, a = i % GE;
                const int jj = i / GE, u = jj % AB;   // the group's jj-th tile, its accumulator
                if (!mbar_wait(&bars->full[pp][s], (i / S) & 1, p.status)) break;
                if (jj >= AB && !mbar_wait(&bars->tempty[pp][a][u], ((jj / AB) & 1) ^ 1, p.status)) break;
                if (i == 0 && !mbar_wait(&bars->q_full, 0, p.status)) break;
                int b, ti;
                locate(tile_of(pp, i), b, ti);
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + lay.k_off + st * kTile * kKeyBytes);
                const uint32_t b_addr = smem_u32(smem + lay.q_off + b * N * kKeyBytes);
                const uint32_t d = tmem_base + (uint32_t)(((pp * GE + a) * AB + u) * N);
#pragma unroll
                for (int k = 0; k < kKeyBytes / 32; ++k)
                    umma_f8(d, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                            k > 0 ? 1u : 0u);
                umma_commit(&bars->empty[pp][s]);
                umma_commit(&bars->tfull[pp][a][u]);
                if (i == 0 && pp == 0 && cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 11] = globaltimer_ns();
            }
            umma_commit(&bars->mma_done[pp]);
            mbar_wait(&bars->mma_done[pp], 0, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Scores only, as the standalone indexer: the candidates are taken
        // from the stored scores after the stream, CTA by CTA.  The group's
        // first tile is also the sample for the thresholds.
        const int ew = warp - kEpiWarp0;
        const int pp = ew / (kMaxGroups * kEpiWarps);
        const int a = (ew / kEpiWarps) % kMaxGroups;
        const int quarter = warp & 3;
        const int gi = pp * kMaxGroups + a;
        const int gbar = kGroupBar0 + gi;
        const int row_in_tile = quarter * 32 + lane;
        const int ng = a < GE ? group_count(pp, a) : 0;
        float *coef = reinterpret_cast<float *>(smem + lay.epi_off) + ew * (17 * T);
        int32_t *qp = reinterpret_cast<int32_t *>(coef + 16 * T);
        const uint32_t acc_col0 = (uint32_t)((pp * GE + a) * AB * N);
        const bool poller = quarter == 0 && lane == 0;
        bool ok = true;
        int cur_b = -1;
        bool polling = false;   // the poller's read of the packed words is in flight
        uint32_t *poll = reinterpret_cast<uint32_t *>(smem + lay.poll_off) + gi * 2 * kMaxRows;
        // This lane's key scale in the group's jn-th tile, loaded one tile
        // ahead (0 past the group's tiles or the sequence).  The scales come
        // from global memory, not through the stage, so a stage is free as
        // soon as its MMA has read it: an epilogue group that is held up (the
        // sample exchange, the thresholds) holds up only its own TMEM
        // accumulators, not the pipeline's ring.
        auto scale_of = [&](int jn) -> float {
            if (jn >= ng) return 0.f;
            int bb, ti2;
            locate(tile_of(pp, jn * GE + a), bb, ti2);
            const int64_t ps = (int64_t)ti2 * kTile + row_in_tile;
            if (ps >= seq_len[bb]) return 0.f;
            bool okr = true;
            const int64_t row = row_of(p, bb, ps, &okr);
            return okr ? __ldcs(cp.k_scale + row) : 0.f;
        };
        float ks_next = scale_of(0);
        int thr_row = -1;   // the row whose threshold this warp computes, once its histogram has arrived
        // Row thr_row's threshold from the histogram copied into shared memory:
        // published (kThr, the packed word), the global histogram cleared for
        // the next call; the last row's warp resets the arrival count and
        // releases kReady.
        auto finish_threshold = [&]() {
            attn::cp_async_wait_all();
            __syncwarp();
            const int r = thr_row;
            thr_row = -1;
            const int64_t n = (int64_t)row_qpos[r] + 1;
            uint32_t t_r = 0xFFFFFFFFu;   // n <= top_k: every key is selected, nothing to capture
            if (n > cp.K) t_r = row_threshold(hist + r * kHistStride, n, cp.K, cp.oversample);
            uint4 *g4 = reinterpret_cast<uint4 *>(cp.sample_hist + r * kHistStride);
            for (int u = lane; u < kHistStride / 4; u += 32) g4[u] = make_uint4(0u, 0u, 0u, 0u);
            if (lane == 0) {
                ctl[kThr + r] = t_r;
                st_relaxed_gpu_u64(reinterpret_cast<uint64_t *>(ctl + kThrPacked) + r, (1ull << 32) | t_r);
                __threadfence();   // this row's words, before the count that the last row's warp reads
                if (atomicAdd(misc + 5, 1u) == (uint32_t)rows - 1) {
                    ctl[kSampleArrive] = 0;   // read by nobody until the next call
                    st_release_gpu(ctl + kReady, 1u);
                }
            }
            __syncwarp();
        };
        for (int j = 0; j < ng || j == 0; ++j) {
            const bool have = j < ng;
            if (thr_row >= 0) finish_threshold();
            const float ks = ks_next;
            ks_next = scale_of(j + 1);
            bool scored = false;
            float sc[kMaxRows] = {0.f, 0.f, 0.f, 0.f};
            uint32_t vis = 0;
            int b = 0;
            int64_t pos = 0;
            if (have && ok) {
                const int i = j * GE + a, s = i % S, st = pp * S + s;
                int ti;
                locate(tile_of(pp, i), b, ti);
                if (b != cur_b) {
                    __syncwarp();
                    for (int u = lane; u < 16 * T; u += 32)
                        coef[u] = __ldg(p.w + (int64_t)b * 16 * T + u) * __ldg(p.q_scale + (int64_t)b * 16 * T + u);
                    for (int u = lane; u < T; u += 32) qp[u] = __ldg(p.q_pos + b * T + u);
                    __syncwarp();
                    cur_b = b;
                }
                const int u = j % AB;
                const uint32_t acc_col = acc_col0 + (uint32_t)(u * N);
                const bool w_ok = mbar_wait(&bars->tfull[pp][a][u], (j / AB) & 1, p.status);
                (void)s;
                (void)st;
                if (__all_sync(0xffffffffu, w_ok)) {
                    scored = true;
                    if (j == 0 && gi == 0 && poller && cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 12] = globaltimer_ns();
                    tc_fence_after();
                    pos = (int64_t)ti * kTile + row_in_tile;
                    const int len = seq_len[b];
                    float *out = p.scores + (int64_t)b * T * p.scores_stride + pos;
#pragma unroll
                    for (int t = 0; t < kMaxRows; ++t) {
                        if (t < T) {
                            float acc[16];
                            tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + acc_col + (uint32_t)(16 * t),
                                      acc);
                            float sum = 0.f;
#pragma unroll
                            for (int h = 0; h < 16; ++h) sum = fmaf(coef[16 * t + h], fmaxf(acc[h], 0.f), sum);
                            const bool visible = pos < len && pos <= qp[t];
                            sc[t] = ks * sum;
                            if (pos < len) out[(int64_t)t * p.scores_stride] = visible ? sc[t] : -INFINITY;
                            if (visible) vis |= 1u << t;
                        }
                    }
                    if (!capturing && j < back_cap) {   // the backlog's keys wait in TMEM
#pragma unroll
                        for (int t = 0; t < T; ++t)
                            tmem_st1(tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                         (uint32_t)(acc_cols + (gi * back_cap + j) * T + t),
                                     float_order_key(sc[t]));
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->tempty[pp][a][u]);
                    if (j == 0) {   // the sample: into the CTA's histogram of each row
#pragma unroll
                        for (int t = 0; t < kMaxRows; ++t)
                            if (t < T)
                                warp_hist_add(hist + (b * T + t) * kHistStride, sample_bin(float_order_key(sc[t])),
                                              (vis >> t) & 1u);
                    }
                } else {
                    ok = false;
                }
            }
            if (j == 0) {
                // ---- sample exchange: CTA histogram -> row histograms -> thresholds
                named_bar_sync(gbar, 128);
                uint32_t *flag = misc + 1 + gi;   // per group: 1 = flushes the CTA, 2 = also computes thresholds
                if (quarter == 0 && lane == 0) {
                    __threadfence_block();
                    *flag = atomicAdd(misc, 1u) == kGroups - 1 ? 1u : 0u;
                    __threadfence_block();
                }
                named_bar_sync(gbar, 128);
                if (*flag) {
                    const int tid = quarter * 32 + lane;
                    for (int u = tid; u < rows * kHistStride; u += 128)
                        if (hist[u]) atomicAdd(cp.sample_hist + u, hist[u]);
                    named_bar_sync(gbar, 128);   // the group's adds, before its poller's release below
                    if (quarter == 0 && lane == 0) {
                        // releases this CTA's adds; the last arrival acquires every CTA's
                        *flag = atom_add_acq_rel_gpu(ctl + kSampleArrive, 1u) == (uint32_t)ncta - 1 ? 2u : 1u;
                        if (cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 7] = globaltimer_ns();
                    }
                    named_bar_sync(gbar, 128);
                    if (*flag == 2u && quarter < rows) {
                        // the last CTA: warp r of the group copies row r's
                        // histogram into shared memory (the CTA's own, already
                        // added in, is free) and goes on with its tiles; it
                        // computes the threshold from the copy a tile later
                        const uint4 *src = reinterpret_cast<const uint4 *>(cp.sample_hist + quarter * kHistStride);
                        uint4 *dst = reinterpret_cast<uint4 *>(hist + quarter * kHistStride);
                        for (int u = lane; u < kHistStride / 4; u += 32) attn::cp_async16(dst + u, src + u);
                        attn::cp_async_commit();
                        thr_row = quarter;
                    }
                }
            }
            // ---- this tile's candidates, once the warp has the thresholds.
            //      Each group's poller copies the packed words into shared
            //      memory asynchronously and looks at the copy one tile later,
            //      so it never waits for it; every warp looks at the CTA's
            //      flag once per tile and switches on its own.
            if (!capturing) {
                if (poller) {
                    if (polling) {
                        attn::cp_async_wait_all();   // (long done)
                        uint64_t w[kMaxRows];
#pragma unroll
                        for (int r = 0; r < kMaxRows; ++r)
                            w[r] = (uint64_t)poll[2 * r] | ((uint64_t)poll[2 * r + 1] << 32);
                        if (all_published(w)) publish(w);
                        polling = false;
                    }
                    if (j + 1 < ng && *reinterpret_cast<volatile uint32_t *>(thr_s + kMaxRows) == 0u) {
                        for (int r2 = 0; r2 < rows; r2 += 2) attn::cp_async16(poll + 2 * r2, packed + r2);
                        attn::cp_async_commit();
                        polling = true;
                    }
                }
                uint32_t seen = lane == 0 ? *reinterpret_cast<volatile uint32_t *>(thr_s + kMaxRows) : 0u;
                if (__shfl_sync(0xffffffffu, seen, 0) != 0u) transition(j);   // the tiles before this one
            }
            if (capturing) {
                uint32_t key[kMaxRows] = {0u, 0u, 0u, 0u}, cand = 0u;
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    key[t] = float_order_key(sc[t]);
                    uint32_t th = 0u;
#pragma unroll
                    for (int rr = 0; rr < kMaxRows; ++rr)
                        if (rr == b * T + t) th = thr[rr];
                    if (scored && ((vis >> t) & 1u) && key[t] >= th) cand |= 1u << t;
                }
                warp_take(b, cand, key, (uint32_t)pos);
            }
        }
        if (thr_row >= 0) finish_threshold();
        if (polling) attn::cp_async_wait_all();
        // ---- after the group's tiles: a warp still without the thresholds
        //      waits for them here, while its backlog is in TMEM
        if (ng > 0 && !capturing) {
            uint32_t okw = 1u;
            const uint32_t seen = lane == 0 ? *reinterpret_cast<volatile uint32_t *>(thr_s + kMaxRows) : 0u;
            if (__shfl_sync(0xffffffffu, seen, 0) == 0u) {
                if (lane == 0) {
                    uint64_t w[kMaxRows];
                    okw = wait_packed(w) ? 1u : 0u;
                    if (okw) publish(w);
                }
                okw = __shfl_sync(0xffffffffu, okw, 0);
            }
            if (okw) transition(ng);
        }
    }
    (void)any_tiles;

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
    __syncthreads();
    if (cp.trace && threadIdx.x == 0) cp.trace[cta * DSA_TRACE_MARKS + 2] = globaltimer_ns();

    // ---- the CTA's candidates: the warps' lists merged into the CTA's
    //      segment of each row's list, in position order
    bool r_ok = true;
    if (threadIdx.x == 0 && n_tiles > 0 && thr_s[kMaxRows] == 0u) {
        r_ok = spin_until_at_least(ctl + kReady, 1u, kWaitLimitNs, p.status);   // (acquire)
        if (r_ok) {
            for (int r = 0; r < rows; ++r) thr_s[r] = ld_relaxed_gpu(ctl + kThr + r);
            thr_s[kMaxRows] = 1u;
            if (cp.trace) cp.trace[cta * DSA_TRACE_MARKS + 1] = globaltimer_ns();
        }
    }
    if (ew_c >= 0 && lane == 0) {
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) wcs[ew_c * kMaxRows + r] = wc[r];
    }
    if (!__syncthreads_and(r_ok)) return;   // the timeout is in the status word; the grid barrier sees it
    // Each epilogue warp places its own list's entries: an entry's place in
    // the segment is the length of the lists of the pipelines before its
    // pipeline (their position ranges are disjoint and in order) plus the
    // entries of its pipeline's eight lists (which interleave: tiles by
    // group, rows within a tile by warp) with a lower position.
    constexpr int kLists = kGroups * kEpiWarps;
    constexpr int kPipeWarps = kMaxGroups * kEpiWarps;   // the epilogue warps of one pipeline
    static_assert(kLists <= 32, "one list length per lane");
    if (ew_c >= 0) {
        for (int r = 0; r < rows; ++r) {
            const uint32_t c_l = lane < kLists ? wcs[lane * kMaxRows + r] : 0u;
            const bool over = __any_sync(0xffffffffu, c_l > (uint32_t)kWarpCap);
            uint32_t incl = c_l;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            const uint32_t total = __shfl_sync(0xffffffffu, incl, kLists - 1);
            const int w0 = e_pp * kPipeWarps;   // the pipeline's first epilogue warp
            const uint32_t pbase = __shfl_sync(0xffffffffu, incl - c_l, w0);
            uint32_t nw[kPipeWarps];
#pragma unroll
            for (int q2 = 0; q2 < kPipeWarps; ++q2) nw[q2] = __shfl_sync(0xffffffffu, c_l, w0 + q2);
            if (!over && total <= (uint32_t)kSegCap) {
                uint2 *seg = cp.lists + ((int64_t)r * cp.NG + cta) * kSegCap;
                uint32_t mine = 0;
#pragma unroll
                for (int q2 = 0; q2 < kPipeWarps; ++q2)
                    if (w0 + q2 == ew_c) mine = nw[q2];
                for (uint32_t i = lane; i < mine; i += 32) {
                    const uint2 ent = wlist(r, ew_c)[i];
                    uint32_t rank = pbase + i;
#pragma unroll
                    for (int q2 = 0; q2 < kPipeWarps; ++q2) {
                        if (w0 + q2 == ew_c) continue;
                        const uint2 *L2 = wlist(r, w0 + q2);
                        uint32_t lo = 0, hi = nw[q2];
                        while (lo < hi) {
                            const uint32_t mid = (lo + hi) >> 1;
                            if (L2[mid].y < ent.y) lo = mid + 1; else hi = mid;
                        }
                        rank += lo;
                    }
                    seg[rank] = ent;
                }
            }
            if (ew_c == 0 && lane == 0) {   // the row's count in this CTA
                const bool ov = over || total > (uint32_t)kSegCap;
                cp.counts[(int64_t)r * cp.NG + cta] = ov ? 0u : total;
                if (total && !ov) atomicAdd(ctl + kTotal + r, total);
                if (ov) atomicOr(ctl + kOverflow, 1u);
            }
        }
    }
    if ((int)threadIdx.x <= kMaxRows) keep[threadIdx.x] = thr_s[threadIdx.x];   // the thresholds and their flag
}

// One slice of the combine of (row bt, KV group g), by the 128 threads of a
// team (tid 0..127) once all `splits` units of that group have written their
// partials: slice `piece` of the group's (head, column) outputs, head-major,
// cut into `splits` near-equal slices.  The operations and their order are
// those of combine_row_cta, so the outputs are identical:
//   M = max(sink, m_j),  w_j = 2^(m_j - M) (0 for an empty split),
//   O = sum_j (v_j w_j) / (2^(sink - M) + sum_j l_j w_j)   in order j = 0, 1, ...
// `st` is team shared memory for the statistics of the slice's heads.
__device__ void combine_piece(const Params &cp, int bt, int g, int piece, int tid, int bar, float *st) {
    const attn::Params &at = cp.at;
    const int hpg = DSA_Q_HEADS / at.G, splits = at.splits;
    const int E = hpg * DSA_V_DIM;
    const int lo = (int)((int64_t)piece * E / splits), hi = (int)((int64_t)(piece + 1) * E / splits);
    const int h_lo = lo / DSA_V_DIM, nh = (hi - 1) / DSA_V_DIM - h_lo + 1;
    float *w = st;                            // [nh][splits] m_j, then the weights w_j
    float *ls = st + hpg * kMaxSplits;        // [nh][splits] l_j
    float *hs = ls + hpg * kMaxSplits;        // [nh][2]: M, L per head
    // this thread's first element's split values, loaded together with the
    // statistics (one round trip to L2 for both)
    float v0[kMaxSplits];
    {
        const int e = lo + tid;
        if (e < hi) {
            const int hh = e / DSA_V_DIM - h_lo, col = e % DSA_V_DIM;
            const int64_t gw = (int64_t)bt * DSA_Q_HEADS + g * hpg + h_lo + hh;
            const float *po = at.part_o + gw * splits * DSA_V_DIM + col;
#pragma unroll
            for (int j = 0; j < kMaxSplits; ++j) v0[j] = j < splits ? __ldcg(po + (int64_t)j * DSA_V_DIM) : 0.f;
        }
    }
    // the heads' split statistics -> weights, M and the denominators
    for (int i = tid; i < nh * splits; i += 128) {
        const int hh = i / splits, j = i % splits;
        const int64_t gw = (int64_t)bt * DSA_Q_HEADS + g * hpg + h_lo + hh;
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(at.part_ml) + gw * splits + j);
        w[i] = ml.x;
        ls[i] = ml.y;
    }
    attn::team_sync(bar);
    {   // per head, one warp: split j on lane j; the max is exact in any
        // order, and lane 0 sums the denominator's terms in split order
        const int wq = tid >> 5, ln = tid & 31;
        for (int hh = wq; hh < nh; hh += 4) {
            const int h = g * hpg + h_lo + hh;
            const float sk = cp.sink ? __ldg(cp.sink + h) * attn::kLog2e : -INFINITY;
            const bool on = ln < splits;
            const float m = on ? w[hh * splits + ln] : -INFINITY;
            float M = m;
#pragma unroll
            for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            M = fmaxf(M, sk);
            const float wj = (M == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M);
            if (on) {
                const float lj = ls[hh * splits + ln];
                w[hh * splits + ln] = wj;
                ls[hh * splits + ln] = wj != 0.f ? __fmul_rn(lj, wj) : 0.f;
            }
            __syncwarp();
            if (ln == 0) {
                float L = (cp.sink && M != -INFINITY) ? exp2f(sk - M) : 0.f;
#pragma unroll 8
                for (int j = 0; j < splits; ++j) L = __fadd_rn(L, ls[hh * splits + j]);
                hs[2 * hh] = M;
                hs[2 * hh + 1] = L;
            }
        }
    }
    attn::team_sync(bar);
    for (int e = lo + tid; e < hi; e += 128) {
        const int hh = e / DSA_V_DIM - h_lo, col = e % DSA_V_DIM;
        const int64_t gw = (int64_t)bt * DSA_Q_HEADS + g * hpg + h_lo + hh;
        const float *po = at.part_o + gw * splits * DSA_V_DIM + col;
        float v[kMaxSplits];
        if (e == lo + tid) {
#pragma unroll
            for (int j = 0; j < kMaxSplits; ++j) v[j] = v0[j];
        } else {
#pragma unroll
            for (int j = 0; j < kMaxSplits; ++j) v[j] = j < splits ? __ldcg(po + (int64_t)j * DSA_V_DIM) : 0.f;
        }
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxSplits; ++j) {
            if (j < splits) {
                const float wj = w[hh * splits + j];
                acc = __fadd_rn(acc, __fmul_rn(wj != 0.f ? v[j] : 0.f, wj));
            }
        }
        const float M = hs[2 * hh], L = hs[2 * hh + 1];
        cp.O[gw * DSA_V_DIM + col] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
        if (cp.lse && col == 0) cp.lse[gw] = (L > 0.f) ? (M + log2f(L)) / attn::kLog2e : -INFINITY;
    }
    attn::team_sync(bar);   // `st` may be reused
}

// Phase 2 (fast): the exact selection of row r from its candidates, into
// `sel` (shared, top_k entries, -1 padded) and, by CTA c == 0, into the
// output.  `work` is shared memory for the list.  Called by all threads;
// thread t < NG passes the length of CTA t's segment of the row (seg_len),
// and keep holds the thresholds kept from phase 1 (see run_indexer_capture).
__device__ void select_from_candidates(const Params &cp, int r, int c, int32_t *sel, uint8_t *work, uint64_t *trace,
                                       uint32_t seg_len, const uint32_t *keep) {
    constexpr int NT = kThreads, NW = NT / 32;
    const int K = cp.K, NG = cp.NG;
    const int lane = lane_id(), warp = warp_id();
    const uint32_t lt = (1u << lane) - 1u;
    auto *sh = reinterpret_cast<topk::Shared<NT> *>(work);
    uint32_t *off = reinterpret_cast<uint32_t *>(work + align128(sizeof(topk::Shared<NT>)));
    uint64_t *copied = reinterpret_cast<uint64_t *>(off + ((NG + 1 + 31) & ~31));   // bulk-copy barriers
    uint2 *list = reinterpret_cast<uint2 *>(copied + 2);   // (order key, position), 16-byte aligned
    uint32_t *wide = reinterpret_cast<uint32_t *>(list + kListCap);   // [kWide] histogram
    uint32_t *bin_keys = wide + kWide;                                // [kSmall] keys of T*'s bin
    int64_t n = (int64_t)__ldg(cp.ix.q_pos + r) + 1;
    if (n > cp.ix.Lmax) n = cp.ix.Lmax;
    if (n < 0) n = 0;
    const int kr = (int)(n < K ? n : K);
    if (n <= K) {
        for (int j = threadIdx.x; j < K; j += NT) sel[j] = j < n ? j : -1;
    } else {
        // the segments, in position order, each padded to an even length so
        // that it moves as one 16-byte-multiple bulk copy; a pad slot gets
        // the entry (key 0, position -1): below every candidate's key (the
        // threshold's, or a finite score's), so it is never selected
        if (threadIdx.x == 0) {
            // the stream's histogram of the row's candidates first, on its own
            // barrier: the k-th key's bin is found from it while the
            // segments are still on their way
            mbar_init(copied, 1);
            mbar_init(copied + 1, 1);
            fence_mbar_init();
            fence_proxy_async_smem();   // earlier use of the area, before the copy overwrites it
            mbar_arrive_expect_tx(copied + 1, kWide * 4u);
            bulk_load(wide, cp.cand_hist + (int64_t)r * kWide, kWide * 4u, copied + 1);
        }
        const uint32_t v = (int)threadIdx.x < NG ? seg_len : 0u;
        const uint32_t vp = (v + 1u) & ~1u;
        uint32_t m;   // entries, pads included
        const uint32_t incl = topk::block_scan<NT>(vp, sh->warp_tmp, &m);
        if (threadIdx.x < NG) off[threadIdx.x] = incl - vp;
        if (threadIdx.x == 0) off[NG] = m;
        fence_proxy_async_smem();   // earlier use of the list area, before the copies overwrite it
        __syncthreads();
        const uint2 *segs = cp.lists + (int64_t)r * NG * kSegCap;
        {   // the expected bytes posted once per warp, before the warp's copies
            // (updates of one mbarrier from many threads serialise)
            uint32_t bytes_w = vp * 8u;   // (0 for threads past the segments)
#pragma unroll
            for (int o = 16; o; o >>= 1) bytes_w += __shfl_xor_sync(0xffffffffu, bytes_w, o);
            if (lane == 0 && bytes_w > 0) mbar_expect_tx(copied, bytes_w);
            __syncwarp();
        }
        if (threadIdx.x < NG && vp > 0)
            bulk_load(list + (incl - vp), segs + (int64_t)threadIdx.x * kSegCap, vp * 8u, copied);
        __syncthreads();   // every expected byte is posted
        if (threadIdx.x == 0) mbar_arrive(copied);
        // ---- the k-th largest key T*, exactly.
        auto is_key = [&](uint32_t j, uint32_t &k) {
            const uint2 e = list[j];
            k = e.x;
            return e.y != 0xFFFFFFFFu;   // not a pad
        };
        // The bin of `wide` (kWide bins, the top one holding the largest
        // keys) that holds the K-th largest key, and the keys above it: 512
        // threads own 8 bins each, from the top.
        auto find_bin = [&]() {
            uint32_t s = 0;
            if (threadIdx.x < kWide / 8)
                for (int i = 0; i < 8; ++i) s += wide[kWide - 1 - 8 * (int)threadIdx.x - i];
            uint32_t tot;
            const uint32_t incl = topk::block_scan<NT>(s, sh->warp_tmp, &tot);
            if (threadIdx.x < kWide / 8 && incl - s < (uint32_t)K && (uint32_t)K <= incl) {
                uint32_t above = incl - s;
                for (int i = 0; i < 8; ++i) {
                    const int b = kWide - 1 - 8 * (int)threadIdx.x - i;
                    if (above + wide[b] >= (uint32_t)K) {
                        sh->bin = b;
                        sh->above = above;
                        break;
                    }
                    above += wide[b];
                }
            }
            __syncthreads();
        };
        // A handful of keys in bin_keys: one warp ranks them; T* is the key
        // with fewer than Krem keys above it and at least Krem at or above.
        auto rank_small = [&](uint32_t n_keys, uint32_t Krem_in, uint32_t &t_out, uint32_t &ties_out) {
            if (warp == 0) {
                const bool valid = (uint32_t)lane < n_keys;
                const uint32_t mine = valid ? bin_keys[lane] : 0u;
                uint32_t gt = 0, ge = 0;
                for (uint32_t q = 0; q < n_keys; ++q) {
                    const uint32_t o = __shfl_sync(0xffffffffu, mine, q);
                    gt += o > mine;
                    ge += o >= mine;
                }
                const uint32_t hit = __ballot_sync(0xffffffffu, valid && gt < Krem_in && Krem_in <= ge);
                const int src = hit ? __ffs(hit) - 1 : 0;
                const uint32_t t_key = __shfl_sync(0xffffffffu, mine, src);
                const uint32_t t_gt = __shfl_sync(0xffffffffu, gt, src);
                if (lane == 0) {
                    sh->base = t_key;
                    sh->above = t_gt;
                }
            }
            __syncthreads();
            t_out = sh->base;
            ties_out = Krem_in - sh->above;
            __syncthreads();
        };
        // Gathers into bin_keys the keys k with pred(k) (any order); their count.
        auto gather_keys = [&](auto pred) {
            if (threadIdx.x == 0) sh->total = 0;
            __syncthreads();
            constexpr uint32_t kG = 4;   // strips whose loads are in flight together
            for (uint32_t jb = threadIdx.x & ~31u; jb < m; jb += kG * NT) {
                uint32_t kk[kG];
                bool tk[kG];
#pragma unroll
                for (uint32_t u = 0; u < kG; ++u) {
                    const uint32_t j = jb + u * NT + lane;
                    kk[u] = 0u;
                    tk[u] = j < m && is_key(j, kk[u]) && pred(kk[u]);
                }
#pragma unroll
                for (uint32_t u = 0; u < kG; ++u) {
                    const uint32_t bits = __ballot_sync(0xffffffffu, tk[u]);
                    if (bits) {
                        uint32_t at = 0;
                        if (lane == 0) at = atomicAdd(&sh->total, (uint32_t)__popc(bits));
                        at = __shfl_sync(0xffffffffu, at, 0) + __popc(bits & lt);
                        if (tk[u] && at < (uint32_t)kSmall) bin_keys[at] = kk[u];
                    }
                }
            }
            __syncthreads();
            const uint32_t n_keys = sh->total;
            __syncthreads();
            return n_keys;
        };
        uint32_t Tstar = 0u, ties = 0u;
        bool found = false;
        // the compaction's layout: 32-entry strips, each warp a run of whole
        // strips, four strips' loads in flight at a time
        const uint32_t strips = (m + 31) / 32, per_w = (strips + NW - 1) / NW;
        const uint32_t s0 = min(strips, (uint32_t)warp * per_w), s1 = min(strips, s0 + per_w);
        constexpr uint32_t kU = 4;
        bool counted = false;   // sh->warp_a / warp_b hold each warp's keys above T* / equal to it
        {   // from the stream's histogram of the row's candidates above its threshold
            const uint32_t thr_r = keep[kMaxRows] ? keep[r] : __ldcg(cp.ctl + kThr + r);
            mbar_wait(copied + 1, 0, cp.ix.status);
            find_bin();
            const int B = sh->bin;
            const uint32_t Kb = (uint32_t)K - sh->above, in_b = wide[B];
            // then the list
            mbar_wait(copied, 0, cp.ix.status);
            if (threadIdx.x < NG && (v & 1u)) list[incl - 1] = make_uint2(0u, 0xFFFFFFFFu);
            __syncthreads();
            if (trace && threadIdx.x == 0) trace[8] = globaltimer_ns();
            if (B < kWide - 1 && in_b <= 32u) {   // not the catch-all bin, and a handful of keys
                // one pass in the compaction's layout: bin B's keys aside, with
                // their warp, and per warp the keys of the bins above B (all
                // above T*, which lies in bin B)
                if (threadIdx.x == 0) sh->total = 0;
                __syncthreads();
                uint32_t above = 0;
                for (uint32_t q = s0; q < s1; q += kU) {
                    uint2 ent[kU];
#pragma unroll
                    for (uint32_t u = 0; u < kU; ++u) {
                        const uint32_t j = (q + u) * 32 + lane;
                        ent[u] = q + u < s1 && j < m ? list[j] : make_uint2(0u, 0xFFFFFFFFu);
                    }
#pragma unroll
                    for (uint32_t u = 0; u < kU; ++u) {
                        const uint2 e = ent[u];
                        const bool key = e.y != 0xFFFFFFFFu && e.x >= thr_r;   // not a pad
                        const uint32_t d = (e.x - thr_r) >> kCandShift;
                        const bool in_bin = key && d == (uint32_t)B;
                        above += __popc(__ballot_sync(0xffffffffu, key && d > (uint32_t)B));
                        const uint32_t bits = __ballot_sync(0xffffffffu, in_bin);
                        if (bits) {
                            uint32_t at = 0;
                            if (lane == 0) at = atomicAdd(&sh->total, (uint32_t)__popc(bits));
                            at = __shfl_sync(0xffffffffu, at, 0) + __popc(bits & lt);
                            if (in_bin && at < 32u) {
                                bin_keys[at] = e.x;
                                bin_keys[kSmall / 2 + at] = (uint32_t)warp;
                            }
                        }
                    }
                }
                if (lane == 0) sh->warp_a[warp] = above;
                __syncthreads();
                const uint32_t n_keys = sh->total;
                if (n_keys == in_b) {   // (always: the histogram counted exactly these keys)
                    rank_small(n_keys, Kb, Tstar, ties);
                    found = true;
                    if ((int)threadIdx.x < NW) {   // each warp's counts, with its keys of bin B
                        uint32_t g2 = sh->warp_a[threadIdx.x], e2 = 0;
                        for (uint32_t i = 0; i < n_keys; ++i)
                            if (bin_keys[kSmall / 2 + i] == threadIdx.x) {
                                g2 += bin_keys[i] > Tstar;
                                e2 += bin_keys[i] == Tstar;
                            }
                        sh->warp_a[threadIdx.x] = g2;
                        sh->warp_b[threadIdx.x] = e2;
                    }
                    counted = true;
                }
            }
        }
        if (!found) {   // the general search: the 12 bits below the keys' common high bits, then the rest
            uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
            for (uint32_t j = threadIdx.x; j < m; j += NT) {
                uint32_t k;
                if (is_key(j, k)) {
                    kmin = min(kmin, k);
                    kmax = max(kmax, k);
                }
            }
            kmin = __reduce_min_sync(0xffffffffu, kmin);
            kmax = __reduce_max_sync(0xffffffffu, kmax);
            if (lane == 0) {
                sh->warp_a[warp] = kmin;
                sh->warp_b[warp] = kmax;
            }
            __syncthreads();
            for (int j = threadIdx.x; j < kWide; j += NT) wide[j] = 0;
            __syncthreads();
            for (int w2 = 0; w2 < NW; ++w2) {
                kmin = min(kmin, sh->warp_a[w2]);
                kmax = max(kmax, sh->warp_b[w2]);
            }
            const int top = kmin == kmax ? 0 : 31 - __clz(kmin ^ kmax);   // highest bit in which keys differ
            const int shift = top > 11 ? top - 11 : 0;
            const uint32_t hi_mask = top >= 31 ? 0u : ~((2u << top) - 1u);   // the bits every key shares
            list_digit_hist<NT>(wide, m, kmin & hi_mask, hi_mask, shift, (uint32_t)kWide, is_key);
            __syncthreads();
            find_bin();
            uint32_t prefix = (kmin & hi_mask) | ((uint32_t)sh->bin << shift);
            uint32_t mask = hi_mask | ((uint32_t)(kWide - 1) << shift);
            uint32_t Krem = (uint32_t)K - sh->above;
            const uint32_t in_bin = wide[sh->bin];
            __syncthreads();
            if (shift > 0) {
                // the keys of T*'s bin into a small buffer (any order), unless too many
                const bool small = in_bin <= (uint32_t)kSmall;
                if (small) gather_keys([&](uint32_t k) { return (k & mask) == prefix; });
                if (small && in_bin <= 32u) {
                    uint32_t t_key, t_ties;
                    rank_small(in_bin, Krem, t_key, t_ties);
                    prefix = t_key;
                    Krem = t_ties;
                } else {
                    // the remaining bits, 11 at a time, over the bin's keys
                    for (int sh2 = shift; sh2 > 0;) {
                        const int w = sh2 > 11 ? 11 : sh2;
                        sh2 -= w;
                        const int nb = 1 << w;
                        for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = 0;
                        __syncthreads();
                        if (small)
                            list_digit_hist<NT>(sh->hist, in_bin, prefix, mask, sh2, (uint32_t)nb,
                                                [&](uint32_t j, uint32_t &k) {
                                                    k = bin_keys[j];
                                                    return true;
                                                });
                        else
                            list_digit_hist<NT>(sh->hist, m, prefix, mask, sh2, (uint32_t)nb, is_key);
                        __syncthreads();
                        topk::find_threshold<NT>(sh, nb, Krem);
                        prefix |= (uint32_t)sh->bin << sh2;
                        mask |= (uint32_t)(nb - 1) << sh2;
                        Krem -= sh->above;
                        __syncthreads();
                    }
                }
            }
            Tstar = prefix;
            ties = Krem;
        }
        if (trace && threadIdx.x == 0) trace[9] = globaltimer_ns();
        // compaction in position order, in the strips: the keys above T* and
        // the first `ties` keys equal to it, each at (keys above before it) +
        // min(equal keys before it, ties); the per-warp counts first (unless
        // the bin search took them), pads never counted
        if (!counted) {
            uint32_t gt = 0, eq = 0;
            for (uint32_t q = s0; q < s1; q += kU) {
                uint2 ent[kU];
#pragma unroll
                for (uint32_t u = 0; u < kU; ++u) {
                    const uint32_t j = (q + u) * 32 + lane;
                    ent[u] = q + u < s1 && j < m ? list[j] : make_uint2(0u, 0xFFFFFFFFu);
                }
#pragma unroll
                for (uint32_t u = 0; u < kU; ++u) {
                    const bool in = ent[u].y != 0xFFFFFFFFu;
                    gt += __popc(__ballot_sync(0xffffffffu, in && ent[u].x > Tstar));
                    eq += __popc(__ballot_sync(0xffffffffu, in && ent[u].x == Tstar));
                }
            }
            if (lane == 0) {
                sh->warp_a[warp] = gt;
                sh->warp_b[warp] = eq;
            }
        }
        __syncthreads();
        uint32_t gb = 0, eb = 0;
        for (int w2 = 0; w2 < warp; ++w2) {
            gb += sh->warp_a[w2];
            eb += sh->warp_b[w2];
        }
        for (uint32_t q = s0; q < s1; q += kU) {
            uint2 ent[kU];
#pragma unroll
            for (uint32_t u = 0; u < kU; ++u) {
                const uint32_t j = (q + u) * 32 + lane;
                ent[u] = q + u < s1 && j < m ? list[j] : make_uint2(0u, 0u);
            }
#pragma unroll
            for (uint32_t u = 0; u < kU; ++u) {
                const uint2 e = ent[u];
                const bool in = q + u < s1 && (q + u) * 32 + lane < m && e.y != 0xFFFFFFFFu;
                const uint32_t bg = __ballot_sync(0xffffffffu, in && e.x > Tstar);
                const uint32_t be = __ballot_sync(0xffffffffu, in && e.x == Tstar);
                const uint32_t g_before = gb + __popc(bg & lt), e_before = eb + __popc(be & lt);
                if (in && e.x > Tstar) sel[g_before + (e_before < ties ? e_before : ties)] = (int32_t)e.y;
                else if (in && e.x == Tstar && e_before < ties) sel[g_before + e_before] = (int32_t)e.y;
                gb += __popc(bg);
                eb += __popc(be);
            }
        }
        for (int j = kr + threadIdx.x; j < K; j += NT) sel[j] = -1;
    }
    __syncthreads();
    if (n > K && threadIdx.x == 0) {
        mbar_inval(copied);
        mbar_inval(copied + 1);
    }
    if (c == 0) {
        int32_t *out = cp.tk.idx + (int64_t)r * K;
        for (int j = threadIdx.x; j < K; j += NT) out[j] = sel[j];
        if (threadIdx.x == 0) cp.tk.count[r] = kr;
    }
}

template <int TQ>
__global__ void __launch_bounds__(kThreads, 1)
dsa_layer_capture_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_ks,
                         const __grid_constant__ CUtensorMap tmap_q, const Params cp) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    __shared__ uint32_t sync_flag;
    __shared__ uint32_t thr_keep[kMaxRows + 1];
    if (threadIdx.x == 0) thr_keep[kMaxRows] = 0u;
    pdl_launch_dependents();   // (the wait comes once the CTA's own set-up is done)
    const uint32_t G = gridDim.x;
    uint32_t *status = cp.ix.status;
    uint32_t *ctl = cp.ctl;
    uint32_t status_at_entry = 0;
    uint64_t *trace = cp.trace ? cp.trace + blockIdx.x * DSA_TRACE_MARKS : nullptr;
    auto mark = [&](int i) {
        if (trace && threadIdx.x == 0) trace[i] = globaltimer_ns();
    };
    // run by every thread right after the dependent-launch wait
    auto after_wait = [&]() {
        status_at_entry = load_status(status);
        if (trace && threadIdx.x == 0) {
            for (int i = 1; i < DSA_TRACE_MARKS; ++i) trace[i] = 0;
            trace[0] = globaltimer_ns();
            trace[13] = clock64();
        }
    };

    // ---- phase 1: key stream, sample, candidates
    run_indexer_capture<TQ>(&tmap_k, &tmap_ks, &tmap_q, cp, smem, blockIdx.x, G, thr_keep, after_wait);
    mark(15);
    if (status_at_entry & kNeedsInitBit) {
        if (threadIdx.x == 0) flag_timeout(status);
        return;
    }
    if (!grid_sync(ctl + kGridArrive, 1 * G, cp.bar, status, &sync_flag)) return;
    mark(3);

    const int rows = cp.rows, C = cp.C;
    // this CTA's row's segment lengths, loaded together with the words that
    // decide the path: the sample was good for every row? (the same answer
    // in every CTA)
    uint32_t seg_len = 0u;
    if ((int)blockIdx.x < rows * C && (int)threadIdx.x < cp.NG)
        seg_len = __ldcg(cp.counts + (int64_t)(blockIdx.x / C) * cp.NG + threadIdx.x);
    bool fast = __ldcg(ctl + kOverflow) == 0u;
    for (int r = 0; r < cp.rows; ++r) {
        const int64_t n = (int64_t)__ldg(cp.ix.q_pos + r) + 1;
        const uint32_t m = __ldcg(ctl + kTotal + r);
        // the list in shared memory holds the candidates and up to one pad per segment
        if (n > cp.K && (m < (uint32_t)cp.K || m + (uint32_t)cp.NG > (uint32_t)kListCap)) fast = false;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {   // read by nobody after phase 1
        ctl[kReady] = 0;
        atomicAdd(cp.path_count + (fast ? 0 : 1), 1u);
    }

    const int G_kv = cp.at.G, splits = cp.at.splits, nt = cp.at.n_teams;
    const attn::TeamSmem teams{smem + (fast ? kSelBytes : 0), (uint32_t)align128(sizeof(attn::Smem))};
    if (fast) {
        // ---- phase 2 (fast): the CTAs of a row that have attention units
        //      select from the row's candidates, attend, then combine.  Unit
        //      u of row r (KV head u / splits, 64-key chunk u % splits) is
        //      taken by team u / C of the row's CTA u % C.
        const int upr = G_kv * splits;   // units of a row (single teams; CTA units when nt > 1, then splits == 1)
        if ((int)blockIdx.x < rows * C && (int)(blockIdx.x % C) < upr) {
            const int r = blockIdx.x / C, c = blockIdx.x % C;
            int32_t *sel = reinterpret_cast<int32_t *>(smem);
            select_from_candidates(cp, r, c, sel, smem + kSelBytes, trace, seg_len, thr_keep);
            mark(4);
            if (nt == 1) {
                const int tm = threadIdx.x >> 7, tid = threadIdx.x & 127;
                if (tm < kTeams) {
                    for (int u = c + tm * C; u < upr; u += kTeams * C) {
                        const int g = u / splits, split = u % splits;
                        attn::attn_unit(cp.at, teams[tm], split, g, r, tid, 1 + tm, sel, true, cp.sink, cp.O, cp.lse);
                        attn::team_sync(1 + tm);   // every thread's stores are done; the count releases them
                        if (splits > 1 && tid == 0) red_release_gpu_add(ctl + kCombine + r * DSA_Q_HEADS + g, 1u);
                    }
                    if (tm == 0) mark(5);
                    // each unit's team then combines one slice of its KV head's
                    // outputs, once every unit of that head has written its partial
                    if (splits > 1) {
                        for (int u = c + tm * C; u < upr; u += kTeams * C) {
                            const int g = u / splits, split = u % splits;
                            bool ok = true;
                            if (tid == 0)
                                ok = spin_until_at_least(ctl + kCombine + r * DSA_Q_HEADS + g, (uint32_t)splits,
                                                         cp.bar.limit_ns, status);
                            if (!named_bar_and(1 + tm, 128, ok)) break;
                            combine_piece(cp, r, g, split, tid, 1 + tm, reinterpret_cast<float *>(&teams[tm]));
                        }
                    }
                }
            } else if ((int)threadIdx.x < nt * 128) {
                // key sets of at most 256: one CTA unit per KV head, no combine
                attn::cta_unit(cp.at, teams, 0, c, r, 1, kUnitBar, cp.sink, cp.O, cp.lse, sel);
                mark(5);
            }
        }
    } else {
        // ---- the general path (as the fused layer-step without the indexer histogram)
        if ((int)blockIdx.x < rows * C) {
            auto *sh = reinterpret_cast<topk::Shared<kThreads> *>(smem);
            uint32_t *cache = reinterpret_cast<uint32_t *>(smem + align128(sizeof(topk::Shared<kThreads>)));
            topk::select_row<kThreads>(cp.tk, sh, cache, blockIdx.x / C, blockIdx.x % C, C, true);
        }
        if (!grid_sync(ctl + kGridArrive, 2 * G, cp.bar, status, &sync_flag)) return;
        {
            const int units = rows * G_kv * splits;
            if ((int)threadIdx.x < kTeams * 128) {
                if (nt == 1) {
                    const int tm = threadIdx.x >> 7;
                    for (int u = blockIdx.x + tm * G; u < units; u += kTeams * G) {
                        const int split = u % splits, g = (u / splits) % G_kv, bt = u / (splits * G_kv);
                        attn::team_unit(cp.at, teams[tm], split, g, bt, threadIdx.x & 127, 1 + tm, cp.sink, cp.O,
                                        cp.lse);
                    }
                } else if ((int)threadIdx.x < nt * 128) {
                    for (int u = blockIdx.x; u < units; u += G) {
                        const int split = u % splits, g = (u / splits) % G_kv, bt = u / (splits * G_kv);
                        attn::cta_unit(cp.at, teams, split, g, bt, 1, kUnitBar, cp.sink, cp.O, cp.lse);
                    }
                }
            } else if ((int)blockIdx.x < rows * C && C > 1) {
                constexpr int kFree = kThreads - kTeams * 128;
                topk::clear_row_share(cp.tk, blockIdx.x / C, blockIdx.x % C, C, false, threadIdx.x - kTeams * 128,
                                      kFree);
            }
        }
        if (!grid_sync(ctl + kGridArrive, 3 * G, cp.bar, status, &sync_flag)) return;
        if ((int)blockIdx.x < rows * C && blockIdx.x % C == 0) topk::reset_row_ctl(cp.tk, blockIdx.x / C, C);
        if (splits > 1)
            for (int gw = blockIdx.x; gw < rows * DSA_Q_HEADS; gw += G)
                attn::combine_row_cta<kThreads>(cp.at.part_o, cp.at.part_ml, gw, splits, cp.sink, cp.O, cp.lse,
                                                reinterpret_cast<float *>(smem));
    }

    // ---- the last CTA out resets the words read by everyone after phase 1
    __syncthreads();
    mark(6);
    if (trace && threadIdx.x == 0) trace[14] = clock64();
    if (threadIdx.x == 0)   // (release: this CTA is done with the words; acquire: the last one sees that)
        sync_flag = atom_add_acq_rel_gpu(ctl + kGridExit, 1u) == G - 1 ? 1u : 0u;
    __syncthreads();
    if (sync_flag) {   // the last CTA out: every other CTA is done with these words
        // (nobody in this launch reads them again; the next launch sees them
        // after this one has completed)
        for (int i = threadIdx.x; i < rows * kWide; i += blockDim.x) cp.cand_hist[i] = 0;
        if (threadIdx.x == 0) {
            ctl[kGridArrive] = 0;
            ctl[kOverflow] = 0;
            for (int r = 0; r < kMaxRows; ++r) {
                ctl[kTotal + r] = 0;
                ctl[kThr + r] = 0;
                ctl[kThrPacked + 2 * r] = 0;
                ctl[kThrPacked + 2 * r + 1] = 0;
            }
            for (int i = 0; i < rows * DSA_Q_HEADS; ++i) ctl[kCombine + i] = 0;
            ctl[kGridExit] = 0;
        }
    }
}

// Whether the one-barrier kernel is launched as a programmatic dependent of
// the previous kernel (on until a launch with both attributes is refused).
static std::atomic<bool> g_pdl_capture{true};
static bool pdl_capture_ok() { return g_pdl_capture.load(); }
static void pdl_capture_off() { g_pdl_capture.store(false); }

// The kernel for T query tokens per sequence (1..kMaxRows).
static const void *capture_kernel_for(int T) {
    switch (T) {
        case 1: return (const void *)dsa_layer_capture_kernel<1>;
        case 2: return (const void *)dsa_layer_capture_kernel<2>;
        case 3: return (const void *)dsa_layer_capture_kernel<3>;
        default: return (const void *)dsa_layer_capture_kernel<4>;
    }
}

}  // namespace capture

// --------------------------------------------------------------- host side
// Largest dynamic shared memory of the capture kernel: the device's opt-in
// maximum less room for the kernel's static shared memory (under 1 KB).
static size_t capture_smem_budget() { return device_info().smem_optin - 1024; }

int plan_capture(int B, int T, int64_t Lmax, int top_k, CapturePlan *plan) {
    using namespace capture;
    const DeviceInfo &dev = device_info();
    plan->ok = false;
    const int rows = B * T;
    if (dev.num_sms <= 0 || rows > kMaxRows || T > kMaxRows || Lmax < kMinContext) return DSA_OK;
    const int grid = dev.num_sms;
    if (grid > kThreads) return DSA_OK;   // the segment offsets are scanned one per thread
    // all CTAs must be resident together: one per SM (occupancy asked once per device)
    static std::mutex mu;
    static int per_sm_cache[64];
    static bool known[64] = {};
    int dev_id = -1;
    cudaError_t e = cudaGetDevice(&dev_id);
    if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) return cuda_fail(e, "cudaGetDevice");
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!known[dev_id]) {
            // all CTAs of every instantiation must be resident together: the least occupancy
            per_sm_cache[dev_id] = 1 << 30;
            for (int t = 1; t <= kMaxRows; ++t) {
                const void *k = capture_kernel_for(t);
                if (int rc = ensure_smem_limit(k, capture_smem_budget(), "cudaFuncSetAttribute(capture)")) return rc;
                int per_sm = 0;
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, capture_smem_budget());
                if (e != cudaSuccess) return cuda_fail(e, "occupancy of the capture kernel");
                per_sm_cache[dev_id] = std::min(per_sm_cache[dev_id], per_sm);
            }
            known[dev_id] = true;
        }
        if (per_sm_cache[dev_id] < 1) return DSA_OK;
    }
    // the shared-memory layouts must fit: phase 1 with at least 3 stages, phase 2's list and attention teams
    if (Layout(3, T, B).total + 1024 > capture_smem_budget()) return DSA_OK;
    const size_t ng = (size_t)grid;   // one candidate segment per CTA and row
    const size_t fast2 = kSelBytes + std::max(align128(sizeof(topk::Shared<kThreads>)) + ((ng + 1 + 31) & ~size_t(31)) * 4 + 16 +
                                                  (size_t)2 * kListCap * 4 + (size_t)(kWide + kSmall) * 4,
                                              kTeams * align128(sizeof(attn::Smem)));
    if (fast2 + 1024 > capture_smem_budget()) return DSA_OK;
    plan->grid = grid;
    plan->rows = rows;
    plan->C = std::max(1, grid / rows);
    plan->NG = (int)ng;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = (off + bytes + 255) & ~size_t(255);
        return at;
    };
    plan->ctl_off = take(kCtlWords * 4);
    plan->hist_off = take((size_t)rows * kHistStride * 4);
    plan->topk_off = take((size_t)rows * topk::scratch_words(plan->C, topk::kListCap, false) * 4);
    plan->cand_hist_off = take((size_t)rows * kWide * 4);
    plan->scratch_bytes = off;
    off = 0;
    plan->counts_off = take((size_t)rows * ng * 4);
    plan->lists_off = take((size_t)rows * ng * kSegCap * 8);
    plan->data_bytes = off;
    plan->ok = true;
    return DSA_OK;
}

int launch_capture(const CapturePlan &plan, const IndexerArgs &ia, const AttnArgs &aa, int top_k, int32_t *idx,
                   int32_t *count, uint8_t *scratch, uint8_t *data, cudaStream_t stream, void *start_event) {
    using namespace capture;
    const size_t budget = capture_smem_budget();
    IndexerLaunch L;
    if (int rc = prepare_indexer(ia, 0, 0, nullptr, budget, &L)) return rc;   // tensor maps and parameters
    // pipeline depth for this kernel's own layout (every row's query block resident, the sample histograms)
    int S = indexer::kMaxStages;
    while (S > 2 && Layout(S, ia.T, ia.B).total + 1024 > budget) --S;
    const size_t smem1 = Layout(S, ia.T, ia.B).total + 1024;
    const size_t ng = (size_t)plan.grid;
    const size_t smem2 = kSelBytes + std::max(align128(sizeof(topk::Shared<kThreads>)) + ((ng + 1 + 31) & ~size_t(31)) * 4 + 16 +
                                                  (size_t)2 * kListCap * 4 + (size_t)(kWide + kSmall) * 4,
                                              kTeams * align128(sizeof(attn::Smem))) +
                         1024;
    const size_t top_fixed = align128(sizeof(topk::Shared<kThreads>));
    const size_t smem = std::max({smem1, smem2, top_fixed + 1024 + 4096});
    if (smem > budget || S < 3) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "capture kernel shared memory does not fit");

    Params cp;
    cp.ix = L.p;
    cp.ix.stages = S;
    cp.ix.groups = indexer::kMaxGroups;
    // TMEM accumulators per epilogue group: four for one query token (2 pipes
    // * 2 groups * 4 * 16 = 256 columns, the backlog beside them), else two
    cp.ix.acc_bufs = ia.T == 1 ? 4 : 2;
    cp.k_scale = static_cast<const float *>(ia.kv->index_k_scale);
    cp.ix.hist_rows = 0;
    cp.ix.q_resident = 1;
    cp.at = attn::make_params(aa);
    if (cp.at.splits > kMaxSplits) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "attention splits above the combine's bound");
    cp.sink = aa.sink;
    cp.O = aa.O;
    cp.lse = aa.lse;
    cp.ctl = reinterpret_cast<uint32_t *>(scratch + plan.ctl_off);
    cp.sample_hist = reinterpret_cast<uint32_t *>(scratch + plan.hist_off);
    cp.counts = reinterpret_cast<uint32_t *>(data + plan.counts_off);
    cp.cand_hist = reinterpret_cast<uint32_t *>(scratch + plan.cand_hist_off);
    cp.lists = reinterpret_cast<uint2 *>(data + plan.lists_off);
    cp.path_count = ia.status + kPathCountWord;
    cp.trace = phase_trace(plan.grid);
    cp.bar = barrier_cfg();
    cp.rows = plan.rows;
    cp.K = top_k;
    cp.C = plan.C;
    cp.NG = plan.NG;
    cp.oversample = 2.0f;
    topk::Params &tp = cp.tk;
    tp.scores = ia.scores;
    tp.stride = ia.scores_stride;
    tp.q_pos = ia.q_pos;
    tp.rows = plan.rows;
    tp.K = top_k;
    tp.C = plan.C;
    tp.idx = idx;
    tp.count = count;
    tp.scratch = reinterpret_cast<uint32_t *>(scratch + plan.topk_off);
    tp.scratch_row_words = topk::scratch_words(plan.C, topk::kListCap, false);
    tp.status = ia.status;
    {
        const int64_t avail = (int64_t)(smem - 1024 - top_fixed) / 4;
        const int64_t chunk = ((ia.Lmax + plan.C - 1) / plan.C + 3) & ~int64_t(3);
        const int64_t cand = std::min<int64_t>(topk::kCandCap, avail / 4) / kWarps * kWarps;
        const int64_t rest = avail - 2 * cand;
        int64_t list = std::min<int64_t>(topk::kListCap, std::max<int64_t>(0, (rest - chunk) / 2));
        if (list < 1024) list = std::min<int64_t>(topk::kListCap, rest / 4);
        tp.smem_list = (int)list;
        tp.cand_cap = (int)cand;
        tp.cache_keys = (int)(rest - 2 * list);
    }
    tp.list_cap = topk::kListCap;
    tp.Lmax = ia.Lmax;
    tp.bar = cp.bar;

    const void *kern = capture_kernel_for(ia.T);
    if (int rc = ensure_smem_limit(kern, smem, "cudaFuncSetAttribute(capture)")) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;   // phase 1's sample and the grid barrier wait on every CTA
    attr[0].val.cooperative = 1;
    // chained after the previous kernel of the stream (programmatic dependent
    // launch): its launch overlaps that kernel's tail; the kernel's first
    // instruction waits for that kernel's completion and memory
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_capture_ok() ? 2 : 1;
    cudaError_t e;
    if (start_event) {
        e = cudaEventRecord(static_cast<cudaEvent_t>(start_event), stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    {
        const CUtensorMap *mk = &L.tmap_k, *mks = &L.tmap_ks, *mq = &L.tmap_q;
        void *args[] = {(void *)mk, (void *)mks, (void *)mq, (void *)&cp};
        e = cudaLaunchKernelExC(&cfg, kern, args);
        if (e != cudaSuccess && cfg.numAttrs == 2) {   // the driver refuses the pair: plain stream order from now on
            (void)cudaGetLastError();
            pdl_capture_off();
            cfg.numAttrs = 1;
            e = cudaLaunchKernelExC(&cfg, kern, args);
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, "capture layer-step launch");
    return DSA_OK;
}

}  // namespace dsa
