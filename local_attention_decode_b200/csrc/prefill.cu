// prefill.cu -- the DSA layer for a block of query tokens of one sequence
// (chunked prefill), with the indexer as one dense fp8 contraction
// [NQ x 16 heads, 128] x [128, keys] on the tensor cores.
//
// What is computed is, for every query token, exactly the decode layer-step
// ("Naive-N0.5-Flash: no full-attention layers, and a runtime built by AI",
// "What 'no full-attention layers' means": every DSA query keeps its own top
// 2,048 of the keys it may see; "Inside a DSA layer": indexer scores, top-k,
// attention over the selected keys).  How:
//   A  threshold  every token's scores over a sample of the keys (every 64th
//                 page, through the indexer kernel), and the sample's c-th
//                 largest score (through the selection kernel) with c chosen so
//                 that about 2 x top_k keys of the whole context score above it;
//   B  capture    (this file) a persistent kernel: per CTA, pairs of 128-key
//                 tiles stay in shared memory while 8-token query blocks stream
//                 through a TMA ring (the 16 MB of query codes of an 8,192-token
//                 chunk stay in L2); per block two tcgen05.mma (M = 128 keys,
//                 N = 8 tokens x 16 heads, K = 128, e4m3 -> fp32 in TMEM); the
//                 epilogue applies ReLU, the head weights, the key scale and the
//                 causal mask and appends every key whose score reaches the
//                 token's threshold to the token's candidate list;
//   C  select     (this file) per token, the exact top-k of its candidates
//                 (ties to the lower position), sorted by position; a token
//                 whose list is short of top_k or overflowed is recorded for the
//                 decode path;
//   D  attention  the sparse attention kernel over all tokens at once.
// The score matrix (8,192 x 1M in the chunked-prefill workload, 34 GB) is
// never written: only the candidates are.
#include <algorithm>
#include <mutex>

#include "indexer_impl.cuh"
#include "kernels.h"
#include "topk_impl.cuh"

namespace dsa {
namespace prefill {

constexpr int kTile = 128;                  // keys per tile (UMMA M)
constexpr int kUnitTiles = 2;               // key tiles held together
constexpr int kQTok = 8;                    // tokens per query block
constexpr int kN = kQTok * 16;              // UMMA N: 8 tokens x 16 heads
constexpr int kKeyBytes = DSA_INDEX_DIM;
constexpr int kQBytes = kN * kKeyBytes;     // 16 KB
constexpr int kMetaFloats = 32;             // per token: 16 head coefficients, threshold, position, pad
constexpr int kMetaBytes = kQTok * kMetaFloats * 4;   // 1 KB
constexpr int kStages = 6;                  // query-block ring
constexpr int kAcc = 2;                     // TMEM accumulator stages (kUnitTiles x kN columns each)
constexpr int kEpiWarps = 4 * kUnitTiles;   // per accumulator stage: lane quarters x tiles
constexpr int kWarps = 2 + kAcc * kEpiWarps;   // producer, MMA issuer, epilogue
constexpr int kThreads = 32 * kWarps;       // 576
constexpr int kKeyStages = 2;               // key units in flight

struct Params {
    const int32_t *block_table;   // one sequence's pages, or null (contiguous rows = positions)
    int32_t max_pages, page_size;
    int64_t num_rows;
    const float *k_scale;         // index-key scales [rows]
    int rows_per_load;            // TMA box height for the keys (page size when pages are smaller than a tile)
    int NQ, nblocks;
    int64_t n_keys;               // keys any token sees (max position + 1)
    int n_units;
    const float *meta;            // [nblocks][8][32]
    const int32_t *block_max;     // [nblocks] the block's largest position (-1: empty)
    uint32_t *cand_cnt;           // [NQ]
    uint2 *cand;                  // [NQ][cap] (order key, position)
    int cap;
    uint32_t *status;
};

struct __align__(8) Bars {
    uint64_t qfull[kStages], qempty[kStages];
    uint64_t kfull[kKeyStages], kempty[kKeyStages];
    uint64_t tfull[kAcc], tempty[kAcc];
    uint64_t done;
};

struct Layout {
    uint32_t k_off, q_off, meta_off, bar_off, tmem_off, total;
    __host__ __device__ Layout() {
        k_off = 0;                                                        // [kKeyStages][kUnitTiles][16 KB]
        q_off = k_off + kKeyStages * kUnitTiles * kTile * kKeyBytes;      // [kStages][16 KB]
        meta_off = q_off + kStages * kQBytes;                             // [kStages][1 KB]
        bar_off = meta_off + kStages * kMetaBytes;
        tmem_off = bar_off + (uint32_t)sizeof(Bars);
        total = tmem_off + 16;
    }
};

__device__ __forceinline__ int64_t key_row(const Params &p, int64_t pos, bool *ok) {
    if (!p.block_table) {
        if (pos >= p.num_rows) { *ok = false; return 0; }
        return pos;
    }
    const int64_t page = pos / p.page_size;
    if (page >= p.max_pages) { *ok = false; return 0; }
    const int32_t id = __ldg(p.block_table + page);
    const int64_t row = (int64_t)id * p.page_size + pos % p.page_size;
    if (id < 0 || row >= p.num_rows) { *ok = false; return 0; }
    return row;
}

// The (unit, block) pairs of a CTA, in the order every role walks them:
// units u = cta, cta + G, ...; for each unit the blocks whose largest
// position reaches the unit's first key.
struct Walk {
    const Params &p;
    int u, b;
    __device__ Walk(const Params &p_, int cta) : p(p_), u(cta), b(-1) {}
    __device__ bool visible(int uu, int bb) const { return (int64_t)__ldg(p.block_max + bb) >= (int64_t)uu * kUnitTiles * kTile; }
    // advance to the next pair; false when the CTA's work is done
    __device__ bool next(int G, bool *new_unit) {
        *new_unit = false;
        for (;;) {
            if (u >= p.n_units) return false;
            for (++b; b < p.nblocks; ++b)
                if (visible(u, b)) return true;
            u += G;
            b = -1;
            *new_unit = true;
        }
    }
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_capture_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_meta, const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    pdl_begin();
    const Layout lay;
    Bars *bars = reinterpret_cast<Bars *>(smem + lay.bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.tmem_off);
    const int warp = warp_id(), lane = lane_id();
    const int G = gridDim.x, cta = blockIdx.x;
    constexpr uint32_t kTmemCols = kAcc * kUnitTiles * kN;   // 512
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->qfull[s], 1);
            mbar_init(&bars->qempty[s], 1 + kEpiWarps);
        }
        for (int s = 0; s < kKeyStages; ++s) {
            mbar_init(&bars->kfull[s], 1);
            mbar_init(&bars->kempty[s], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(&bars->tfull[a], 1);
            mbar_init(&bars->tempty[a], kEpiWarps);
        }
        mbar_init(&bars->done, 1);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_meta);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            Walk w(p, cta);
            bool new_unit;
            int i = 0, k = -1, issued = 0;
            const int R = p.rows_per_load;
            bool ok = true;
            while (ok && w.next(G, &new_unit)) {
                if (i == 0 || new_unit) {   // the unit's key tiles into the next key stage
                    ++k;
                    const int ks = k % kKeyStages;
                    if (k >= kKeyStages && !mbar_wait(&bars->kempty[ks], ((k / kKeyStages) & 1) ^ 1, p.status)) break;
                    mbar_arrive_expect_tx(&bars->kfull[ks], kUnitTiles * kTile * kKeyBytes);
                    uint8_t *kdst = smem + lay.k_off + ks * kUnitTiles * kTile * kKeyBytes;
                    for (int j = 0; j < kUnitTiles * kTile / R; ++j) {
                        const int64_t pos = (int64_t)w.u * kUnitTiles * kTile + j * R;
                        bool rok = true;
                        int64_t row = 0;
                        if (pos < p.n_keys) {
                            row = key_row(p, pos, &rok);
                            if (!rok) { flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX); row = 0; }
                        }
                        tma_load_2d(kdst + j * R * kKeyBytes, &tmap_k, &bars->kfull[ks], 0, (int32_t)row);
                    }
                }
                const int s = i % kStages;
                if (i >= kStages && !mbar_wait(&bars->qempty[s], ((i / kStages) & 1) ^ 1, p.status)) break;
                mbar_arrive_expect_tx(&bars->qfull[s], kQBytes + kMetaBytes);
                tma_load_2d(smem + lay.q_off + s * kQBytes, &tmap_q, &bars->qfull[s], 0, w.b * kN);
                tma_load_2d(smem + lay.meta_off + s * kMetaBytes, &tmap_meta, &bars->qfull[s], 0, w.b * kQTok);
                ++i;
                ++issued;
            }
            // drain: no copy left in flight into shared memory
            for (int j = max(0, issued - kStages); j < issued; ++j) mbar_wait(&bars->qfull[j % kStages], (j / kStages) & 1, p.status);
            for (int j = max(0, k - kKeyStages + 1); j <= k; ++j)
                mbar_wait(&bars->kfull[j % kKeyStages], (j / kKeyStages) & 1, p.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3_f32(kTile, kN);
            Walk w(p, cta);
            bool new_unit;
            int i = 0, k = -1;
            while (w.next(G, &new_unit)) {
                if (i == 0 || new_unit) {
                    if (k >= 0) umma_commit(&bars->kempty[k % kKeyStages]);   // the previous unit's keys are read
                    ++k;
                    if (!mbar_wait(&bars->kfull[k % kKeyStages], (k / kKeyStages) & 1, p.status)) break;
                }
                const int s = i % kStages, a = i % kAcc;
                if (!mbar_wait(&bars->qfull[s], (i / kStages) & 1, p.status)) break;
                if (i >= kAcc && !mbar_wait(&bars->tempty[a], ((i / kAcc) & 1) ^ 1, p.status)) break;
                tc_fence_after();
                const uint32_t b_addr = smem_u32(smem + lay.q_off + s * kQBytes);
#pragma unroll
                for (int t = 0; t < kUnitTiles; ++t) {
                    const uint32_t a_addr =
                        smem_u32(smem + lay.k_off + ((k % kKeyStages) * kUnitTiles + t) * kTile * kKeyBytes);
                    const uint32_t d = tmem_base + (uint32_t)((a * kUnitTiles + t) * kN);
#pragma unroll
                    for (int kk = 0; kk < kKeyBytes / 32; ++kk)
                        umma_f8(d, umma_desc_k_sw128(a_addr + 32 * kk), umma_desc_k_sw128(b_addr + 32 * kk), idesc,
                                kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars->qempty[s]);
                umma_commit(&bars->tfull[a]);
                ++i;
            }
            if (k >= 0) umma_commit(&bars->kempty[k % kKeyStages]);
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, p.status);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int e = warp - 2;                  // 0 .. 15
        const int a = e / kEpiWarps;             // accumulator stage = parity of the pair index
        const int tile = (e / 4) % kUnitTiles;
        const int quarter = warp & 3;            // TMEM lanes this warp may read
        const uint32_t lt = (1u << lane) - 1u;
        Walk w(p, cta);
        bool new_unit;
        int i = 0;
        float ks = 0.f;
        int64_t kp = 0;
        bool key_ok = false;
        int cur_u = -1;
        while (w.next(G, &new_unit)) {
            const int my = i % kAcc == a;
            if (!my) { ++i; continue; }
            const int s = i % kStages;
            if (w.u != cur_u) {   // this unit's key: its position and scale (from global, read once)
                cur_u = w.u;
                kp = ((int64_t)w.u * kUnitTiles + tile) * kTile + quarter * 32 + lane;
                key_ok = kp < p.n_keys;
                if (key_ok) {
                    bool rok = true;
                    const int64_t row = key_row(p, kp, &rok);
                    key_ok = rok;
                    ks = rok ? __ldg(p.k_scale + row) : 0.f;
                }
            }
            bool wok = mbar_wait(&bars->tfull[a], (i / kAcc) & 1, p.status) &&
                       mbar_wait(&bars->qfull[s], (i / kStages) & 1, p.status);
            if (!__all_sync(0xffffffffu, wok)) break;
            tc_fence_after();
            const float *meta = reinterpret_cast<const float *>(smem + lay.meta_off + s * kMetaBytes);
            const uint32_t col0 = (uint32_t)((a * kUnitTiles + tile) * kN);
#pragma unroll 1
            for (int t = 0; t < kQTok; ++t) {
                float acc[16];
                tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + col0 + (uint32_t)(16 * t), acc);
                const float *m = meta + t * kMetaFloats;
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < 16; ++h) sum = fmaf(m[h], fmaxf(acc[h], 0.f), sum);
                const float thr = m[16];
                const int64_t pos_t = (int64_t)__float_as_int(m[17]);
                const float score = ks * sum;
                const bool cand = key_ok && kp <= pos_t && score >= thr;
                const uint32_t bm = __ballot_sync(0xffffffffu, cand);
                if (bm) {
                    const int tok = w.b * kQTok + t;
                    uint32_t base = 0;
                    if (lane == 0) base = atomicAdd(p.cand_cnt + tok, (uint32_t)__popc(bm));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (cand) {
                        const uint32_t slot = base + __popc(bm & lt);
                        if (slot < (uint32_t)p.cap)
                            p.cand[(int64_t)tok * p.cap + slot] = make_uint2(float_order_key(score), (uint32_t)kp);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->tempty[a]);
                mbar_arrive(&bars->qempty[s]);
            }
            ++i;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------- metadata
// Per token: w x q_scale for the 16 heads, the threshold, the position (as
// its bit pattern); per block of 8 tokens, the largest position.
__global__ void prefill_meta_kernel(const float *w, const float *q_scale, const float *thr, const int32_t *q_pos,
                                    int NQ, int nblocks, float *meta, int32_t *block_max) {
    pdl_begin();
    const int tok = blockIdx.x * blockDim.y + threadIdx.y, c = threadIdx.x;   // 32 x 8 threads
    if (tok >= nblocks * kQTok) return;
    float v = 0.f;
    if (tok < NQ) {
        if (c < 16) v = __ldg(w + (int64_t)tok * 16 + c) * __ldg(q_scale + (int64_t)tok * 16 + c);
        else if (c == 16) v = __ldg(thr + tok);
        else if (c == 17) v = __int_as_float(__ldg(q_pos + tok));
    } else if (c == 17) {
        v = __int_as_float(-1);
    }
    meta[(int64_t)tok * kMetaFloats + c] = v;
    if (c == 0 && (tok % kQTok) == 0) {
        int32_t mx = -1;
        for (int t = tok; t < tok + kQTok && t < NQ; ++t) mx = max(mx, __ldg(q_pos + t));
        block_max[tok / kQTok] = mx;
    }
}

// ------------------------------------------------------- sample positions
// The sample: every s-th logical page (page size ps) of the sequence.  Its
// block table, and per token the last visible sample position.
__global__ void prefill_sample_kernel(const int32_t *block_table, int ps, int s, int n_sample_pages, int B_rep,
                                      const int32_t *q_pos, int NQ, int32_t *sample_table, int32_t *sample_pos) {
    pdl_begin();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n_sample_pages * B_rep) {
        const int j = i % n_sample_pages;
        sample_table[i] = block_table ? __ldg(block_table + (int64_t)j * s) : j * s;
    }
    if (i < NQ) {
        const int64_t p = __ldg(q_pos + i);
        const int64_t span = (int64_t)s * ps;
        const int64_t J = p / span;                 // sample pages wholly or partly at or before p
        const int64_t part = p - J * span + 1;      // positions of page J that p sees (page J starts at J * span)
        int64_t visible = J * ps + (part < ps ? part : ps);
        const int64_t cap = (int64_t)n_sample_pages * ps;
        if (visible > cap) visible = cap;
        sample_pos[i] = (int32_t)(visible - 1);
    }
}

// ---------------------------------------------------------------- select
// One CTA per token: the exact top-k of its candidates (score descending,
// ties to the lower position), sorted by position.  A token whose list
// overflowed, or holds fewer than min(top_k, n) keys, is appended to the
// redo list instead.
constexpr int kSelThreads = 512;

__global__ void __launch_bounds__(kSelThreads)
prefill_select_kernel(const uint32_t *cand_cnt, const uint2 *cand, int cap, const int32_t *q_pos, int64_t Lmax,
                      int K, int32_t *idx, int32_t *count, uint32_t *redo_n, int32_t *redo) {
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_begin();
    constexpr int NT = kSelThreads;
    const int tok = blockIdx.x, t = threadIdx.x;
    auto *sh = reinterpret_cast<topk::Shared<NT> *>(smem);
    uint32_t *lkey = reinterpret_cast<uint32_t *>(smem + ((sizeof(topk::Shared<NT>) + 15) & ~size_t(15)));
    uint32_t *lpos = lkey + cap;
    int32_t *sel = reinterpret_cast<int32_t *>(lpos + cap);   // [K] then sorted in place
    int64_t n = (int64_t)__ldg(q_pos + tok) + 1;
    if (n > Lmax) n = Lmax;
    int32_t *out = idx + (int64_t)tok * K;
    const uint32_t m = __ldcg(cand_cnt + tok);
    if (n <= K) {   // every visible key
        for (int j = t; j < K; j += NT) out[j] = j < n ? j : -1;
        if (t == 0) count[tok] = (int32_t)(n > 0 ? n : 0);
        return;
    }
    if (m > (uint32_t)cap || m < (uint32_t)K) {   // the decode path redoes this token
        for (int j = t; j < K; j += NT) out[j] = -1;
        if (t == 0) {
            count[tok] = 0;
            redo[atomicAdd(redo_n, 1u)] = tok;
        }
        return;
    }
    for (uint32_t j = t; j < m; j += NT) {
        const uint2 e = __ldcg(cand + (int64_t)tok * cap + j);
        lkey[j] = e.x;
        lpos[j] = e.y;
    }
    __syncthreads();
    // k-th largest key
    uint32_t prefix = 0, mask = 0, Krem = (uint32_t)K;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0), nb = pass == 2 ? 1024 : 2048;
        for (int b = t; b < nb; b += NT) sh->hist[b] = 0;
        __syncthreads();
        list_digit_hist<NT>(sh->hist, m, prefix, mask, shift, (uint32_t)nb, [&](uint32_t j, uint32_t &k) { k = lkey[j]; return true; });
        __syncthreads();
        topk::find_threshold<NT>(sh, nb, Krem);
        prefix |= (uint32_t)sh->bin << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        Krem -= sh->above;
        __syncthreads();
    }
    const uint32_t Tstar = prefix, ties = Krem;
    // among the keys equal to T*, the `ties` lowest positions: the ties-th
    // smallest position P* by a radix select on the positions (skipped when
    // every equal key is taken)
    uint32_t eq = 0;
    for (uint32_t j = t; j < m; j += NT) eq += lkey[j] == Tstar;
    uint32_t n_eq;
    topk::block_scan<NT>(eq, sh->warp_tmp, &n_eq);
    uint32_t Pstar = 0xFFFFFFFFu;
    if (n_eq > ties) {
        // the ties-th smallest = the (n_eq - ties + 1)-th largest of the complemented positions
        uint32_t pprefix = 0, pmask = 0, Kp = n_eq - ties + 1;
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0), nb = pass == 2 ? 1024 : 2048;
            for (int b = t; b < nb; b += NT) sh->hist[b] = 0;
            __syncthreads();
            list_digit_hist<NT>(sh->hist, m, pprefix, pmask, shift, (uint32_t)nb, [&](uint32_t j, uint32_t &v) {
                v = ~lpos[j];
                return lkey[j] == Tstar;
            });
            __syncthreads();
            topk::find_threshold<NT>(sh, nb, Kp);
            pprefix |= (uint32_t)sh->bin << shift;
            pmask |= (uint32_t)(nb - 1) << shift;
            Kp -= sh->above;
            __syncthreads();
        }
        Pstar = ~pprefix;   // positions <= P* among the equal keys: exactly `ties` of them
    }
    // compaction (unordered), then a bitonic sort of the K positions
    uint32_t *nsel = &sh->total;
    if (t == 0) *nsel = 0;
    __syncthreads();
    for (uint32_t j = t; j < m; j += NT) {
        const uint32_t k = lkey[j];
        if (k > Tstar || (k == Tstar && lpos[j] <= Pstar)) sel[atomicAdd(nsel, 1u)] = (int32_t)lpos[j];
    }
    __syncthreads();
    int P2 = 1;
    while (P2 < K) P2 <<= 1;
    for (int j = K + t; j < P2; j += NT) sel[j] = 0x7FFFFFFF;   // padding sorts last
    __syncthreads();
    for (int size = 2; size <= P2; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int j = t; j < P2 / 2; j += NT) {
                const int lo = 2 * j - (j & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int32_t x = sel[lo], y = sel[hi];
                if ((x > y) == up) {
                    sel[lo] = y;
                    sel[hi] = x;
                }
            }
            __syncthreads();
        }
    for (int j = t; j < K; j += NT) out[j] = sel[j];
    if (t == 0) count[tok] = K;
}

}  // namespace prefill
}  // namespace dsa

// --------------------------------------------------------------- host side
namespace dsa {

constexpr int kSampleStride = 64;   // every 64th page of keys is in the sample
constexpr int kCandCap = 8192;      // candidates a token may hold
constexpr int kAttnChunkTokens = 1024;

static size_t al(size_t x) { return (x + 255) & ~size_t(255); }

int plan_prefill_capture(int NQ, int64_t Lmax, int top_k, PrefillPlan *pl) {
    pl->ok = false;
    if (NQ < 64 || NQ % 16 != 0 || Lmax < 4096 || top_k > DSA_MAX_TOPK) return DSA_OK;
    const DeviceInfo &dev = device_info();
    if (dev.num_sms <= 0) return DSA_OK;
    if (prefill::Layout().total + 1024 > dev.smem_optin) return DSA_OK;
    pl->NQ = NQ;
    pl->K = top_k;
    pl->Lmax = Lmax;
    pl->nblocks = (NQ + prefill::kQTok - 1) / prefill::kQTok;
    pl->B_rep = NQ / 16;
    pl->s = kSampleStride;
    pl->max_ps = 256;                                   // largest page size this path takes
    pl->Ls_cap = ((Lmax / kSampleStride + pl->max_ps + 127) / 128) * 128;   // sample positions, any page size <= 256
    pl->cap = kCandCap;
    pl->attn_chunk = std::min(NQ, kAttnChunkTokens);
    // the sample's selection (B_rep sequences of 16 tokens), c chosen per call
    if (int rc = plan_topk(pl->B_rep, 16, pl->Ls_cap, DSA_MAX_TOPK, &pl->tp)) return rc;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off = al(off + bytes); return at; };
    pl->topk_scratch = take(pl->tp.scratch_bytes);   // self-cleaning: first, at a fixed offset
    pl->sample_table = take((size_t)pl->B_rep * (pl->Ls_cap / 16 + 1) * 4);
    pl->sample_pos = take((size_t)NQ * 4);
    pl->sample_scores = take((size_t)NQ * pl->Ls_cap * 4);
    pl->sample_idx = take((size_t)NQ * DSA_MAX_TOPK * 4);
    pl->sample_cnt = take((size_t)NQ * 4);
    pl->thr = take((size_t)NQ * 4);
    pl->meta = take((size_t)pl->nblocks * prefill::kQTok * prefill::kMetaFloats * 4);
    pl->block_max = take((size_t)pl->nblocks * 4);
    pl->cand_cnt = take((size_t)NQ * 4);
    pl->cand = take((size_t)NQ * pl->cap * 8);
    pl->idx = take((size_t)NQ * top_k * 4);
    pl->count = take((size_t)NQ * 4);
    pl->redo_n = take(16);
    pl->redo = take((size_t)NQ * 4);
    const int splits = attn_splits(top_k);
    pl->part_o = take((size_t)pl->attn_chunk * DSA_Q_HEADS * splits * DSA_V_DIM * 4);
    pl->part_ml = take((size_t)pl->attn_chunk * DSA_Q_HEADS * splits * 2 * 4);
    pl->total = off;
    pl->ok = true;
    return DSA_OK;
}

int run_prefill_capture(const PrefillPlan &pl, const PrefillArgs &a, uint8_t *ws, cudaStream_t s,
                        int32_t *redo_host, int *n_redo) {
    using namespace prefill;
    const dsa_kv_t *kv = a.kv;
    const int NQ = pl.NQ, K = pl.K;
    const int ps = kv->block_table ? kv->page_size : 128;
    if (ps > pl.max_ps) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "prefill capture path: page size %d > %d", ps, pl.max_ps);
    const int64_t n_pages = (a.Lmax + ps - 1) / ps;
    const int n_sample_pages = (int)((n_pages + pl.s - 1) / pl.s);
    const int64_t Ls = (int64_t)n_sample_pages * ps;
    if (Ls > pl.Ls_cap) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "prefill sample exceeds its plan");
    int32_t *sample_table = reinterpret_cast<int32_t *>(ws + pl.sample_table);
    int32_t *sample_pos = reinterpret_cast<int32_t *>(ws + pl.sample_pos);
    float *sample_scores = reinterpret_cast<float *>(ws + pl.sample_scores);
    float *thr = reinterpret_cast<float *>(ws + pl.thr);
    float *meta = reinterpret_cast<float *>(ws + pl.meta);
    int32_t *block_max = reinterpret_cast<int32_t *>(ws + pl.block_max);
    uint32_t *cand_cnt = reinterpret_cast<uint32_t *>(ws + pl.cand_cnt);
    uint2 *cand = reinterpret_cast<uint2 *>(ws + pl.cand);
    int32_t *idx = a.idx_out ? a.idx_out : reinterpret_cast<int32_t *>(ws + pl.idx);
    int32_t *count = a.count_out ? a.count_out : reinterpret_cast<int32_t *>(ws + pl.count);
    uint32_t *redo_n = reinterpret_cast<uint32_t *>(ws + pl.redo_n);
    int32_t *redo = reinterpret_cast<int32_t *>(ws + pl.redo);
    cudaError_t e;

    // ---- A: thresholds from the sample (every s-th page)
    {
        const int n = std::max(n_sample_pages * pl.B_rep, NQ);
        e = launch_kernel(prefill_sample_kernel, dim3((n + 255) / 256), dim3(256), 0, s, kv->block_table, ps, pl.s,
                          n_sample_pages, pl.B_rep, a.q_pos, NQ, sample_table, sample_pos);
        if (e != cudaSuccess) return cuda_fail(e, "prefill sample launch");
        dsa_kv_t skv = *kv;
        skv.block_table = sample_table;
        skv.max_pages = n_sample_pages;
        skv.page_size = ps;
        IndexerArgs ia{a.q8, a.q_scale, a.w, &skv, sample_pos, pl.B_rep, 16, Ls, sample_scores, Ls, a.status};
        if (int rc = launch_indexer(ia, s)) return rc;
        const int c = (int)std::min<int64_t>(DSA_MAX_TOPK, (2 * (int64_t)K * Ls + a.Lmax - 1) / a.Lmax + 16);
        TopkPlan tp;
        if (int rc = plan_topk(pl.B_rep, 16, Ls, c, &tp)) return rc;
        if (tp.scratch_bytes > pl.tp.scratch_bytes) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "prefill sample scratch");
        if (int rc = launch_topk(tp, sample_scores, Ls, sample_pos, c, reinterpret_cast<int32_t *>(ws + pl.sample_idx),
                                 reinterpret_cast<int32_t *>(ws + pl.sample_cnt),
                                 reinterpret_cast<uint32_t *>(ws + pl.topk_scratch), a.status, s, thr))
            return rc;
    }
    // ---- B: the contraction with the candidate filter
    e = launch_kernel(prefill_meta_kernel, dim3(pl.nblocks), dim3(32, kQTok), 0, s, a.w, a.q_scale, (const float *)thr,
                      a.q_pos, NQ, pl.nblocks, meta, block_max);
    if (e == cudaSuccess) e = cudaMemsetAsync(cand_cnt, 0, (size_t)NQ * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(redo_n, 0, 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill metadata");
    {
        const int R = kv->block_table ? std::min(kv->page_size, kTile) : kTile;
        CUtensorMap tk, tq, tm;
        {
            uint64_t dims[2] = {(uint64_t)kKeyBytes, (uint64_t)kv->num_rows};
            uint64_t strides[1] = {(uint64_t)kKeyBytes};
            uint32_t box[2] = {(uint32_t)kKeyBytes, (uint32_t)R};
            if (int rc = make_tensor_map("prefill keys", &tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kv->index_k, dims,
                                         strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return rc;
        }
        {
            uint64_t dims[2] = {(uint64_t)kKeyBytes, (uint64_t)NQ * 16};
            uint64_t strides[1] = {(uint64_t)kKeyBytes};
            uint32_t box[2] = {(uint32_t)kKeyBytes, (uint32_t)kN};
            if (int rc = make_tensor_map("prefill queries", &tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q8, dims, strides,
                                         box, CU_TENSOR_MAP_SWIZZLE_128B))
                return rc;
        }
        {
            uint64_t dims[2] = {(uint64_t)kMetaFloats, (uint64_t)pl.nblocks * kQTok};
            uint64_t strides[1] = {(uint64_t)kMetaFloats * 4};
            uint32_t box[2] = {(uint32_t)kMetaFloats, (uint32_t)kQTok};
            if (int rc = make_tensor_map("prefill metadata", &tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, meta, dims,
                                         strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
                return rc;
        }
        Params p;
        p.block_table = kv->block_table;
        p.max_pages = kv->max_pages;
        p.page_size = kv->page_size;
        p.num_rows = kv->block_table ? kv->num_rows : std::min<int64_t>(kv->num_rows, kv->seq_stride);
        p.k_scale = kv->index_k_scale;
        p.rows_per_load = R;
        p.NQ = NQ;
        p.nblocks = pl.nblocks;
        p.n_keys = a.Lmax;
        p.n_units = (int)((a.Lmax + kUnitTiles * kTile - 1) / (kUnitTiles * kTile));
        p.meta = meta;
        p.block_max = block_max;
        p.cand_cnt = cand_cnt;
        p.cand = cand;
        p.cap = pl.cap;
        p.status = a.status;
        const size_t smem = Layout().total + 1024;
        if (int rc = ensure_smem_limit((const void *)prefill_capture_kernel, smem, "cudaFuncSetAttribute(prefill)"))
            return rc;
        const int grid = std::min(device_info().num_sms, p.n_units);
        e = launch_kernel(prefill_capture_kernel, dim3(grid), dim3(kThreads), smem, s, tk, tq, tm, p);
        if (e != cudaSuccess) return cuda_fail(e, "prefill capture launch");
    }
    // ---- C: per-token exact selection
    {
        int P2 = 1;
        while (P2 < K) P2 <<= 1;
        const size_t smem = ((sizeof(topk::Shared<kSelThreads>) + 15) & ~size_t(15)) + (size_t)pl.cap * 8 + (size_t)P2 * 4;
        if (int rc = ensure_smem_limit((const void *)prefill_select_kernel, smem, "cudaFuncSetAttribute(prefill select)"))
            return rc;
        e = launch_kernel(prefill_select_kernel, dim3(NQ), dim3(kSelThreads), smem, s, (const uint32_t *)cand_cnt,
                          (const uint2 *)cand, pl.cap, a.q_pos, a.Lmax, K, idx, count, redo_n, redo);
        if (e != cudaSuccess) return cuda_fail(e, "prefill select launch");
    }
    // ---- D: attention of every token, in chunks of tokens
    for (int t0 = 0; t0 < NQ; t0 += pl.attn_chunk) {
        const int T = std::min(pl.attn_chunk, NQ - t0);
        AttnArgs aa;
        aa.Q = a.Q + (size_t)t0 * DSA_Q_HEADS * DSA_QK_DIM;
        aa.kv = kv;
        aa.idx = idx + (size_t)t0 * K;
        aa.count = count + t0;
        aa.idx_stride = K;
        aa.q_pos = nullptr;
        aa.window = 0;
        aa.B = 1;
        aa.T = T;
        aa.max_keys = K;
        aa.sink = a.sink;
        aa.sm_scale = a.sm_scale;
        aa.O = a.O + (size_t)t0 * DSA_Q_HEADS * DSA_V_DIM;
        aa.lse = a.lse ? a.lse + (size_t)t0 * DSA_Q_HEADS : nullptr;
        aa.part_o = reinterpret_cast<float *>(ws + pl.part_o);
        aa.part_ml = reinterpret_cast<float *>(ws + pl.part_ml);
        aa.status = a.status;
        aa.padded = 1;   // rows are full length, -1 past the selection
        if (int rc = launch_attention(aa, s)) return rc;
    }
    // ---- the tokens whose candidate list did not hold their selection
    uint32_t nr = 0;
    e = cudaMemcpyAsync(&nr, redo_n, 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "prefill redo count");
    *n_redo = (int)std::min<uint32_t>(nr, (uint32_t)NQ);
    if (*n_redo > 0) {
        e = cudaMemcpy(redo_host, redo, (size_t)*n_redo * 4, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "prefill redo list");
    }
    return DSA_OK;
}

}  // namespace dsa
