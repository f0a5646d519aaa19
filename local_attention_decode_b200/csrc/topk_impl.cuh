// topk_impl.cuh -- the top-k selection of one query row by a group of CTAs
// (device code shared by the standalone selection kernel and the fused
// layer-step kernel).
//
// For a row of n visible scores: the min(top_k, n) positions with the largest
// scores, equal scores broken toward the lower position ("Naive-N0.5-Flash:
// no full-attention layers, and a runtime built by AI", sections "What 'no
// full-attention layers' means" -- argsort(...)[..., :index_top_k] -- and "How
// much of this did AI actually build?" -- the stable-tie argsort).
//
// Exact radix select on the order-preserving 32-bit image of each score,
// giving the threshold key T* and the number `ties` of keys equal to T* that
// are taken; the output is, in increasing position order, every position with
// key > T* and the first `ties` positions with key == T*.  C CTAs share a row,
// each owning a contiguous slice.  Two paths:
//
// General path (select_row; 11 + 11 + 10-bit digits), slices kept in shared
// memory when they fit:
//   digit 1     the CTAs add their slices' 2048-bin histograms of the top 11
//               bits into the row's global histogram and meet at a barrier;
//   digit 2     the same exchange for the next 11 bits of the keys in the
//               threshold bin; in the same pass each warp keeps its candidates
//               (keys at or above the threshold bin) in shared memory;
//   list        every CTA appends its keys that share the threshold's top 22
//               bits, with their positions, to the row's candidate list and
//               publishes how many of its keys lie above them; one barrier;
//   digit 3     each CTA loads the (short) list and finishes the select on it
//               alone; its output offset is the earlier CTAs' counts above the
//               22-bit bin plus the list entries that lie before its slice.
//               When the list does not fit in shared memory (many keys share
//               the 22-bit bin, e.g. heavy ties), digit 3 is exchanged like the
//               others, and so are the per-CTA (greater, equal) counts at T*;
//   emission    each warp compacts its candidates (or its part of the slice)
//               with ballots, from its own offset in the row's output.
//
// One-barrier path (select_row_hist; fused kernel): the indexer has already
// built the row's histogram of bits 30..20 (eight bins per octave) of the
// non-negative keys.  The threshold bin comes from it; every key at or above
// that bin goes, with its position, to a row-wide list; after one barrier each
// CTA resolves the remaining 20 bits on the list in shared memory, takes its
// offset from the list entries before its slice, and emits its candidates.
//
// The output is a pure function of the scores.  The row's scratch words are
// zeroed again for the next call (by the last CTA to leave, or, in the fused
// kernel, by clear_row_share / reset_row_ctl after a grid barrier).
#pragma once

#include "common.cuh"

namespace dsa {
namespace topk {

constexpr int kBins = 2048;                 // largest digit: 11 bits
constexpr int kUnroll = 8;                  // independent loads in flight per thread
constexpr int kUnrollGlobal = 16;           // the same, for slices read from global memory
constexpr int kListCap = 12288;             // candidate-list entries per row (global scratch)
constexpr int kSmemList = 4096;             // candidate-list entries a CTA takes into shared memory
constexpr int kCandCap = 8192;              // per-warp candidates a CTA keeps in shared memory, in all

// Per-row scratch (u32 words), used when C > 1 or when the first histogram is
// produced by the indexer:
//   [kHist1, +2048) [kHist2, +2048) [kHist3, +1024)  digit histograms
//   [kCnt, +2C)      per-CTA (greater, equal) counts at T* (exchange path)
//   [kCnt+2C, +C)    per-CTA counts of keys above the 22-bit threshold bin
//   ctl_base(C):     [0] barrier arrivals, [1] CTAs done, [2] list length,
//                    [3] a CTA's candidates overflowed its shared memory,
//                    [4] list length of the one-barrier path (select_row_hist)
//   list_base(C):    list_cap keys, then list_cap positions
//   histi_base(C, list_cap), only when the indexer builds it: kHistIWords
//                    words, bits 30..20 of the non-negative keys (2048 bins)
//                    and the count of negative keys
constexpr int kHist1 = 0, kHist2 = 2048, kHist3 = 4096, kCnt = 5120;
constexpr int kHistIWords = 2052;
__host__ __device__ constexpr int ctl_base(int C) { return kCnt + 3 * C; }
constexpr int kCtlWords = 5;
__host__ __device__ constexpr int list_base(int C) { return (ctl_base(C) + kCtlWords + 3) & ~3; }
__host__ __device__ constexpr int histi_base(int C, int list_cap) { return list_base(C) + 2 * list_cap; }
__host__ __device__ constexpr int scratch_words(int C, int list_cap, bool histi = false) {
    return histi_base(C, list_cap) + (histi ? kHistIWords : 0);
}

struct Params {
    const float *scores;
    int64_t stride;
    const int32_t *q_pos;
    int rows, K, C;
    int32_t *idx;
    int32_t *count;
    uint32_t *scratch;
    int scratch_row_words;
    uint32_t *status;
    int cache_keys;        // keys of the slice kept in shared memory
    int list_cap;          // list entries in the row's global scratch
    int smem_list;         // list entries that fit in shared memory after the cache (<= list_cap)
    int cand_cap;          // candidate entries in shared memory after the list (a multiple of NT / 32)
    int64_t Lmax;
    BarrierCfg bar;        // time limit (and injected extra arrivals) of the row barriers
    float *kth = nullptr;  // optional [rows]: the k-th largest visible score (-inf when n <= K)
    int var_c = 0;         // CTAs per row in proportion to the rows' lengths (see row_of_cta); C is then the largest
};


template <int NT>
struct alignas(16) Shared {
    uint32_t hist[kBins];
    uint32_t warp_tmp[NT / 32];
    uint32_t warp_a[NT / 32];
    uint32_t warp_b[NT / 32];
    uint32_t warp_c[NT / 32];
    int bin;
    uint32_t above;
    uint32_t total;
    uint32_t ok;
    uint32_t base;
};

// Length-proportional split of gridDim.x CTAs over the rows (rows <= grid):
// row r gets 1 + floor(n_r * (grid - rows) / sum n) CTAs, n_r = its visible
// keys.  Every CTA computes the same split and finds its (row, c, C_r); a CTA
// past the last row gets row = -1.  All NT threads call it.
template <int NT>
__device__ void row_of_cta(const Params &p, Shared<NT> *sh, int *row, int *c, int *C) {
    constexpr int NW = NT / 32;
    const int rows = p.rows, G = gridDim.x;
    // total visible keys
    uint64_t tot = 0;
    for (int r = threadIdx.x; r < rows; r += NT) {
        int64_t n = (int64_t)__ldg(p.q_pos + r) + 1;
        n = n > p.Lmax ? p.Lmax : (n < 0 ? 0 : n);
        tot += (uint64_t)n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    __shared__ uint64_t s_tot[NW];
    __shared__ int s_row, s_c, s_C;
    if (lane_id() == 0) s_tot[warp_id()] = tot;
    if (threadIdx.x == 0) s_row = -1;
    __syncthreads();
    if (warp_id() == 0) {
        uint64_t t = lane_id() < NW ? s_tot[lane_id()] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        const uint64_t extra = (uint64_t)(G - rows);
        // prefix of the per-row counts, 32 rows at a time
        int base = 0;
        for (int r0 = 0; r0 < rows; r0 += 32) {
            const int r = r0 + lane_id();
            int cr = 0;
            if (r < rows) {
                int64_t n = (int64_t)__ldg(p.q_pos + r) + 1;
                n = n > p.Lmax ? p.Lmax : (n < 0 ? 0 : n);
                cr = 1 + (t > 0 ? (int)((uint64_t)n * extra / t) : 0);
            }
            int incl = cr;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane_id() >= o) incl += u;
            }
            const int first = base + incl - cr;
            if (r < rows && (int)blockIdx.x >= first && (int)blockIdx.x < first + cr) {
                s_row = r;
                s_c = (int)blockIdx.x - first;
                s_C = cr;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    *row = s_row;
    *c = s_c;
    *C = s_C;
}

// Inclusive block scan of one value per thread (all NT threads); returns the
// inclusive prefix and writes the block total to *total.
template <int NT>
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t *warp_tmp, uint32_t *total) {
    constexpr int NW = NT / 32;
    const int lane = lane_id(), warp = warp_id();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < NW ? warp_tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < NW) warp_tmp[lane] = w;
    }
    __syncthreads();
    uint32_t add = warp > 0 ? warp_tmp[warp - 1] : 0;
    *total = warp_tmp[NW - 1];
    __syncthreads();
    return v + add;
}

// Threshold bin of sh->hist[0..nbins): the bin b with above(b) < K <= above(b) + h[b],
// above(b) = number of keys in bins > b.  Result in sh->bin / sh->above, the
// histogram's total in sh->total (bin 0, above 0 when K exceeds the total).
// nbins is 1024 or 2048.  One warp searches: each lane sums a run of nbins / 32
// bins, a suffix scan over the lanes finds the run, the warp then splits that run.
template <int NT>
__device__ __forceinline__ void find_threshold(Shared<NT> *sh, int nbins, uint32_t K) {
    if (warp_id() == 0) {
        const int lane = lane_id();
        const int per = nbins >> 5;
        const uint32_t *h = sh->hist + lane * per;
        uint32_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        for (int j = 0; j < per; j += 4) {   // rotated: no bank conflicts
            s0 += h[(j + lane) & (per - 1)];
            s1 += h[(j + 1 + lane) & (per - 1)];
            s2 += h[(j + 2 + lane) & (per - 1)];
            s3 += h[(j + 3 + lane) & (per - 1)];
        }
        const uint32_t s = (s0 + s1) + (s2 + s3);
        uint32_t incl = s;   // keys in this lane's run and all higher runs
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += u;
        }
        const uint32_t above_run = incl - s;
        const uint32_t total = __shfl_sync(0xffffffffu, incl, 0);
        const uint32_t hit = __ballot_sync(0xffffffffu, above_run < K && K <= incl);
        if (lane == 0) {
            sh->total = total;
            sh->bin = 0;
            sh->above = 0;
        }
        if (hit) {
            const int L = __ffs(hit) - 1;
            const uint32_t base = __shfl_sync(0xffffffffu, above_run, L);
            const int q = per >> 5;   // bins of run L per lane: 2 or 1
            const int b0 = L * per + lane * q;
            uint32_t t = 0;
            for (int j = 0; j < q; ++j) t += sh->hist[b0 + j];
            uint32_t inc2 = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t u = __shfl_down_sync(0xffffffffu, inc2, o);
                if (lane + o < 32) inc2 += u;
            }
            uint32_t run = base + inc2 - t;   // keys above this lane's bins
            for (int j = q - 1; j >= 0; --j) {
                const uint32_t hb = sh->hist[b0 + j];
                if (run < K && K <= run + hb) {
                    sh->bin = b0 + j;
                    sh->above = run;
                }
                run += hb;
            }
        }
    }
    __syncthreads();
}

// Loads nb (<= kBins) histogram words from global memory into sh->hist, all
// loads of a thread in flight together.
template <int NT>
__device__ __forceinline__ void load_hist(Shared<NT> *sh, const uint32_t *g, int nb) {
    constexpr int kPer = (kBins + NT - 1) / NT;
    uint32_t v[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int j = u * NT + threadIdx.x;
        v[u] = j < nb ? __ldcg(g + j) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int j = u * NT + threadIdx.x;
        if (j < nb) sh->hist[j] = v[u];
    }
    __syncthreads();
}

// Sum of a[0 .. upto) (upto <= 32), returned in every lane of the warp.
__device__ __forceinline__ uint32_t warp_sum_prefix(const uint32_t *a, int upto) {
    uint32_t v = lane_id() < upto ? a[lane_id()] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Barrier among the C CTAs of a row: arrive, then wait (bounded) until
// `target` (+ the injected extra, normally 0) arrivals have been counted.
template <int NT>
__device__ bool row_barrier(Shared<NT> *sh, uint32_t *bar, uint32_t target, const BarrierCfg &cfg,
                            uint32_t *status) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        const bool ok = spin_until_at_least(bar, target + cfg.extra, cfg.limit_ns, status);
        __threadfence();
        sh->ok = ok ? 1u : 0u;
    }
    __syncthreads();
    return sh->ok != 0;
}

// The slice [0, len) split into one part per warp, each a whole number of
// 32-key groups: [wlo, whi).
template <int NT>
__device__ __forceinline__ void warp_part(int64_t len, int64_t *wlo, int64_t *whi) {
    constexpr int NW = NT / 32;
    const int64_t sub = ((len + NW - 1) / NW + 31) & ~int64_t(31);
    const int64_t a = (int64_t)warp_id() * sub;
    *wlo = a < len ? a : len;
    *whi = a + sub < len ? a + sub : len;
}

// Calls fn(j, valid, k) for the keys j of this warp's part [wlo, whi), 32
// consecutive keys per call, in position order (all lanes call fn together).
// Keys cached in shared memory are read one group at a time (compact code);
// keys read from global memory are fetched kUnrollGlobal groups at a time.
template <class KeyAt, class Fn>
__device__ __forceinline__ void warp_walk(int64_t wlo, int64_t whi, bool cached, const uint32_t *cache,
                                          KeyAt key_at, Fn fn) {
    const int lane = lane_id();
    if (cached) {
#pragma unroll 1
        for (int64_t j0 = wlo; j0 < whi; j0 += 32) {
            const int64_t j = j0 + lane;
            const bool valid = j < whi;
            fn(j, valid, valid ? cache[j] : 0u);
        }
    } else {
        for (int64_t base = wlo; base < whi; base += 32 * kUnrollGlobal) {
            uint32_t kk[kUnrollGlobal];
#pragma unroll
            for (int u = 0; u < kUnrollGlobal; ++u) {
                const int64_t j = base + u * 32 + lane;
                kk[u] = j < whi ? key_at(j) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kUnrollGlobal; ++u) fn(base + u * 32 + lane, base + u * 32 + lane < whi, kk[u]);
        }
    }
}

// Per-warp counts over the slice: keys > hi_k into sh->warp_a[warp], keys in
// [lo_k, hi_k] into sh->warp_b[warp].  Ends with a __syncthreads().
template <int NT, class KeyAt>
__device__ __forceinline__ void warp_counts(Shared<NT> *sh, int64_t len, bool cached, const uint32_t *cache,
                                            KeyAt key_at, uint32_t lo_k, uint32_t hi_k) {
    int64_t wlo, whi;
    warp_part<NT>(len, &wlo, &whi);
    uint32_t g = 0, e = 0;
    warp_walk(wlo, whi, cached, cache, key_at, [&](int64_t, bool valid, uint32_t k) {
        g += valid && k > hi_k;
        e += valid && k >= lo_k && k <= hi_k;
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane_id() == 0) {
        sh->warp_a[warp_id()] = g;
        sh->warp_b[warp_id()] = e;
    }
    __syncthreads();
}

// This CTA's part of the output, after warp_counts(T, T): in position order,
// its keys > T and its keys == T whose row-wide rank among the keys == T
// (eq_before + rank within the CTA) is below `ties`, written from
// out[out_pos] on (never at or past K).
template <int NT, class KeyAt>
__device__ __forceinline__ void emit_slice(Shared<NT> *sh, int64_t len, int64_t lo, bool cached, const uint32_t *cache,
                                           KeyAt key_at, uint32_t T, uint32_t ties, uint32_t eq_before,
                                           uint32_t out_pos, int32_t *out, int K) {
    const int warp = warp_id(), lane = lane_id();
    uint32_t eq_seen = eq_before + warp_sum_prefix(sh->warp_b, warp);
    if (sh->warp_a[warp] == 0 && (sh->warp_b[warp] == 0 || eq_seen >= ties)) return;   // nothing selected here
    int64_t wlo, whi;
    warp_part<NT>(len, &wlo, &whi);
    const uint32_t cta_eq = eq_before < ties ? eq_before : ties;
    uint32_t o = out_pos + warp_sum_prefix(sh->warp_a, warp) + ((eq_seen < ties ? eq_seen : ties) - cta_eq);
    const uint32_t lt = (1u << lane) - 1u;
    warp_walk(wlo, whi, cached, cache, key_at, [&](int64_t j, bool valid, uint32_t k) {
        const bool is_eq = valid && k == T;
        const uint32_t em = __ballot_sync(0xffffffffu, is_eq);
        const bool sel = (valid && k > T) || (is_eq && eq_seen + __popc(em & lt) < ties);
        const uint32_t sm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const uint32_t at = o + __popc(sm & lt);
            if (at < (uint32_t)K) out[at] = (int32_t)(lo + j);
        }
        o += __popc(sm);
        eq_seen += __popc(em);
    });
}

// Selection of row `row` by CTA c of the C CTAs that share it.  All NT
// threads of the CTA call this.  `cache` holds p.cache_keys keys, then
// 2 * p.smem_list list words, then 2 * p.cand_cap candidate words.
// defer_clear: leave the row's scratch words for clear_row_share and
// reset_row_ctl (called once every CTA of the row is past the selection).
// status_at_entry: the status word as the kernel read it at entry; when it
// says the scratch needs re-initialisation the row is not selected (the
// timeout is flagged again) before any cross-CTA word is touched.
template <int NT>
__device__ void select_row(const Params &p, Shared<NT> *sh, uint32_t *cache, int row, int c, int C,
                           bool defer_clear = false, uint32_t status_at_entry = 0u) {
    const int K = p.K;
    int64_t n = (int64_t)__ldg(p.q_pos + row) + 1;
    if (n > p.Lmax) {   // a position beyond the scores buffer: flag it, select within the buffer
        if (c == 0 && threadIdx.x == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
        n = p.Lmax;
    }
    int32_t *out = p.idx + (int64_t)row * K;
    const float *src = p.scores + (int64_t)row * p.stride;
    uint32_t *rs = C > 1 ? p.scratch + (int64_t)row * p.scratch_row_words : nullptr;
    uint32_t *ctl = rs ? rs + ctl_base(C) : nullptr;

    if (n <= K) {   // every visible position is selected (same decision in all CTAs of the row)
        if (c == 0) {
            for (int j = threadIdx.x; j < K; j += NT) out[j] = j < n ? j : -1;
            if (threadIdx.x == 0) {
                p.count[row] = (int32_t)(n > 0 ? n : 0);
                if (p.kth) p.kth[row] = -INFINITY;
            }
        }
        return;
    }

    const int64_t chunk = ((n + C - 1) / C + 3) & ~int64_t(3);
    const int64_t lo = n < (int64_t)c * chunk ? n : (int64_t)c * chunk;
    const int64_t hi = n < lo + chunk ? n : lo + chunk;
    const int64_t len = hi - lo;
    const bool cached = len <= p.cache_keys;
    uint32_t *lkey = cache + p.cache_keys, *lpos = lkey + p.smem_list;
    constexpr int NW = NT / 32;
    const int warp = warp_id(), lane = lane_id();
    const uint32_t lt = (1u << lane) - 1u;
    const int seg = p.cand_cap / NW;   // candidate entries per warp
    uint32_t *wkey = lpos + p.smem_list + warp * seg, *wpos = wkey + p.cand_cap;

    // scores may have been written earlier in the same kernel: read them through L2 (no .nc loads)
    auto key_at = [&](int64_t j) -> uint32_t { return cached ? cache[j] : float_order_key(__ldcg(src + lo + j)); };
    if (cached) {
        for (int64_t base = 0; base < len; base += (int64_t)kUnroll * NT) {
            float v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * NT + threadIdx.x;
                v[u] = j < len ? __ldcg(src + lo + j) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * NT + threadIdx.x;
                if (j < len) cache[j] = float_order_key(v[u]);
            }
        }
    }
    __syncthreads();
    // Histogram (into sh->hist) of the slice keys that share `prefix` under
    // `mask`, by the nb-bin digit at `shift`.
    auto slice_hist = [&](uint32_t prefix, uint32_t mask, int shift, int nb) {
        for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = 0;
        __syncthreads();
        int64_t wlo, whi;
        warp_part<NT>(len, &wlo, &whi);
        warp_walk(wlo, whi, cached, cache, key_at, [&](int64_t, bool valid, uint32_t k) {
            warp_hist_add(sh->hist, (k >> shift) & (nb - 1), valid && (k & mask) == prefix);
        });
        __syncthreads();
    };
    uint32_t barrier_no = 0;
    // Adds this CTA's histogram into the row's global one at g, waits for the
    // other CTAs of the row, and loads the row's histogram back.
    auto exchange_hist = [&](uint32_t *g, int nb) -> bool {
        for (int j = threadIdx.x; j < nb; j += NT)
            if (sh->hist[j]) atomicAdd(g + j, sh->hist[j]);
        if (!row_barrier<NT>(sh, ctl, ++barrier_no * C, p.bar, p.status)) return false;
        load_hist<NT>(sh, g, nb);
        return true;
    };

    // ---- digit 1
    slice_hist(0u, 0u, 21, kBins);
    if (C > 1 && (status_at_entry & kNeedsInitBit)) {
        if (threadIdx.x == 0) flag_timeout(p.status);
        return;
    }
    if (C > 1 && !exchange_hist(rs + kHist1, kBins)) return;
    find_threshold<NT>(sh, kBins, (uint32_t)K);
    uint32_t prefix = (uint32_t)sh->bin << 21, mask = 0xFFE00000u, Krem = (uint32_t)K - sh->above;
    __syncthreads();
    // Narrows (prefix, mask, Krem) by the nb-bin digit at `shift`, from sh->hist.
    auto take_digit = [&](int nb, int shift) {
        find_threshold<NT>(sh, nb, Krem);
        prefix |= (uint32_t)sh->bin << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        Krem -= sh->above;
        __syncthreads();
    };

    // ---- digit 2, over the whole row; in the same pass each warp keeps, in
    //      position order, its candidates: the keys at or above the threshold bin
    for (int j = threadIdx.x; j < kBins; j += NT) sh->hist[j] = 0;
    __syncthreads();
    int64_t wlo, whi;
    warp_part<NT>(len, &wlo, &whi);
    uint32_t wc = 0;
    warp_walk(wlo, whi, cached, cache, key_at, [&](int64_t j, bool valid, uint32_t k) {
        warp_hist_add(sh->hist, (k >> 10) & (kBins - 1), valid && (k & mask) == prefix);
        const bool cand = valid && k >= prefix;
        const uint32_t cm = __ballot_sync(0xffffffffu, cand);
        if (cand) {
            const uint32_t slot = wc + __popc(cm & lt);
            if (slot < (uint32_t)seg) {
                wkey[slot] = k;
                wpos[slot] = (uint32_t)(lo + j);
            }
        }
        wc += __popc(cm);
    });
    if (lane == 0) sh->warp_a[warp] = wc;
    __syncthreads();
    if (C > 1 && threadIdx.x == 0) {
        bool over = false;
        for (int w = 0; w < NW; ++w) over |= sh->warp_a[w] > (uint32_t)seg;
        if (over) atomicOr(ctl + 3, 1u);
    }
    if (C > 1 && !exchange_hist(rs + kHist2, kBins)) return;
    take_digit(kBins, 10);
    // every CTA's candidates fit: (read after the exchange, the same in every CTA)
    const bool cand_ok = C > 1 && seg > 0 && __ldcg(ctl + 3) == 0u;

    // ---- the candidate list: every key of the row whose top 22 bits are the
    //      threshold's, with its position; each CTA publishes its count of keys
    //      above them
    bool use_list = false;
    uint32_t m = 0;
    if (C > 1) {
        const uint32_t hi22 = prefix | ~mask;
        uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
        if (cand_ok) {
            const uint32_t wc = sh->warp_a[warp];
            uint32_t a = 0, e = 0;
            for (uint32_t i = lane; i < wc; i += 32) {
                a += wkey[i] > hi22;
                e += (wkey[i] & mask) == prefix;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, o);
                e += __shfl_xor_sync(0xffffffffu, e, o);
            }
            if (lane == 0) {
                sh->warp_c[warp] = a;
                sh->warp_b[warp] = e;
            }
        } else {
            warp_counts<NT>(sh, len, cached, cache, key_at, prefix, hi22);   // above into warp_a, in-bin into warp_b
            if (lane == 0) sh->warp_c[warp] = sh->warp_a[warp];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t above = 0, mine = 0;
            for (int w = 0; w < NW; ++w) {
                above += sh->warp_c[w];
                mine += sh->warp_b[w];
            }
            rs[kCnt + 2 * C + c] = above;
            sh->base = mine ? atomicAdd(ctl + 2, mine) : 0u;
        }
        __syncthreads();
        if (sh->warp_b[warp]) {   // append this warp's keys of the 22-bit bin
            uint32_t at = sh->base + warp_sum_prefix(sh->warp_b, warp);
            auto put = [&](bool in, uint32_t k, uint32_t pos) {
                const uint32_t bm = __ballot_sync(0xffffffffu, in);
                if (in) {
                    const uint32_t slot = at + __popc(bm & lt);
                    if (slot < (uint32_t)p.list_cap) {
                        gkey[slot] = k;
                        gpos[slot] = pos;
                    }
                }
                at += __popc(bm);
            };
            if (cand_ok) {
                const uint32_t wc = sh->warp_a[warp];
                for (uint32_t i0 = 0; i0 < wc; i0 += 32) {
                    const uint32_t i = i0 + lane;
                    const uint32_t k = i < wc ? wkey[i] : 0u;
                    put(i < wc && (k & mask) == prefix, k, i < wc ? wpos[i] : 0u);
                }
            } else {
                int64_t wlo, whi;
                warp_part<NT>(len, &wlo, &whi);
                warp_walk(wlo, whi, cached, cache, key_at, [&](int64_t j, bool valid, uint32_t k) {
                    put(valid && (k & mask) == prefix, k, (uint32_t)(lo + j));
                });
            }
        }
        if (!row_barrier<NT>(sh, ctl, ++barrier_no * C, p.bar, p.status)) return;
        m = __ldcg(ctl + 2);
        use_list = m <= (uint32_t)p.smem_list;
        if (use_list) {
            const uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
            for (uint32_t base = 0; base < m; base += 4 * NT) {
                uint32_t kv[4], pv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t j = base + u * NT + threadIdx.x;
                    kv[u] = j < m ? __ldcg(gkey + j) : 0u;
                    pv[u] = j < m ? __ldcg(gpos + j) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t j = base + u * NT + threadIdx.x;
                    if (j < m) {
                        lkey[j] = kv[u];
                        lpos[j] = pv[u];
                    }
                }
            }
            __syncthreads();
        }
    }

    // ---- digit 3: on the list, or over the row
    if (use_list) {
        for (int j = threadIdx.x; j < 1024; j += NT) sh->hist[j] = 0;
        __syncthreads();
        list_digit_hist<NT>(sh->hist, m, prefix, mask, 0, 1024u, [&](uint32_t j, uint32_t &k) { k = lkey[j]; return true; });
        __syncthreads();
    } else {
        slice_hist(prefix, mask, 0, 1024);
        if (C > 1 && !exchange_hist(rs + kHist3, 1024)) return;
    }
    take_digit(1024, 0);
    const uint32_t Tstar = prefix;
    const uint32_t ties = Krem;   // keys equal to T* that are taken (>= 1)
    if (p.kth && c == 0 && threadIdx.x == 0)   // the k-th largest score itself (the inverse of float_order_key)
        p.kth[row] = __uint_as_float((Tstar & 0x80000000u) ? (Tstar & 0x7FFFFFFFu) : ~Tstar);

    // ---- this CTA's offset in the row's output
    uint32_t gt_before = 0, eq_before = 0;
    if (use_list) {
        // earlier CTAs: all their keys above the 22-bit bin, and their list entries > T* / == T*
        uint32_t a = 0, e = 0;
        for (int j = threadIdx.x; j < c; j += NT) a += __ldcg(rs + kCnt + 2 * C + j);
        for (uint32_t j = threadIdx.x; j < m; j += NT)
            if ((int64_t)lpos[j] < lo) {
                a += lkey[j] > Tstar;
                e += lkey[j] == Tstar;
            }
        block_scan<NT>(a, sh->warp_tmp, &gt_before);
        block_scan<NT>(e, sh->warp_tmp, &eq_before);
    }
    const uint32_t out_pos = gt_before + min(eq_before, ties);

    // ---- emission
    if (cand_ok && use_list) {
        // from the candidates: per-warp counts at T*, then ordered compaction
        const uint32_t wc = sh->warp_a[warp];
        uint32_t g = 0, e = 0;
        for (uint32_t i = lane; i < wc; i += 32) {
            g += wkey[i] > Tstar;
            e += wkey[i] == Tstar;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) {
            sh->warp_b[warp] = g;
            sh->warp_c[warp] = e;
        }
        __syncthreads();
        uint32_t eq_seen = eq_before + warp_sum_prefix(sh->warp_c, warp);
        const uint32_t cta_eq = eq_before < ties ? eq_before : ties;
        uint32_t o = out_pos + warp_sum_prefix(sh->warp_b, warp) + ((eq_seen < ties ? eq_seen : ties) - cta_eq);
        if (g || (e && eq_seen < ties)) {
            for (uint32_t i0 = 0; i0 < wc; i0 += 32) {
                const uint32_t i = i0 + lane;
                const uint32_t k = i < wc ? wkey[i] : 0u;
                const bool is_eq = i < wc && k == Tstar;
                const uint32_t em = __ballot_sync(0xffffffffu, is_eq);
                const bool sel = (i < wc && k > Tstar) || (is_eq && eq_seen + __popc(em & lt) < ties);
                const uint32_t sm = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                    const uint32_t at = o + __popc(sm & lt);
                    if (at < (uint32_t)K) out[at] = (int32_t)wpos[i];
                }
                o += __popc(sm);
                eq_seen += __popc(em);
            }
        }
    } else {
        warp_counts<NT>(sh, len, cached, cache, key_at, Tstar, Tstar);
        if (!use_list && C > 1) {   // exchange the per-CTA (greater, equal) counts at T*
            uint32_t *cnt = rs + kCnt;
            if (threadIdx.x == 0) {
                uint32_t g = 0, e = 0;
                for (int w = 0; w < NW; ++w) {
                    g += sh->warp_a[w];
                    e += sh->warp_b[w];
                }
                cnt[2 * c] = g;
                cnt[2 * c + 1] = e;
            }
            if (!row_barrier<NT>(sh, ctl, ++barrier_no * C, p.bar, p.status)) return;
            uint32_t a = 0, e = 0;
            for (int j = threadIdx.x; j < c; j += NT) {
                a += __ldcg(cnt + 2 * j);
                e += __ldcg(cnt + 2 * j + 1);
            }
            block_scan<NT>(a, sh->warp_tmp, &gt_before);
            block_scan<NT>(e, sh->warp_tmp, &eq_before);
        }
        emit_slice<NT>(sh, len, lo, cached, cache, key_at, Tstar, ties, eq_before, gt_before + min(eq_before, ties), out, K);
    }
    if (c == 0 && threadIdx.x == 0) p.count[row] = K;

    // ---- the last CTA of the row to leave clears the row's words for the next call
    if (defer_clear) return;
    __syncthreads();
    if (C > 1) {
        if (threadIdx.x == 0) {
            __threadfence();
            sh->ok = atomicAdd(ctl + 1, 1u) == (uint32_t)C - 1;
        }
        __syncthreads();
        if (sh->ok) {
            __threadfence();
            for (int j = threadIdx.x; j < ctl_base(C); j += NT) rs[j] = 0;
            const uint32_t used = m < (uint32_t)p.list_cap ? m : (uint32_t)p.list_cap;
            uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
            for (uint32_t j = threadIdx.x; j < used; j += NT) {
                gkey[j] = 0;
                gpos[j] = 0;
            }
            if (threadIdx.x == 0) {
                for (int j = 0; j < kCtlWords; ++j) ctl[j] = 0;
            }
        }
    }
}

// One-barrier selection of row `row` by CTA c of C (C > 1), for a row whose
// score histogram the indexer has already built in the row's scratch
// (at histi_base: bits 30..20 of the non-negative keys, eight bins per octave, and
// the count of negative keys).  Each thread holds up to kHistRegs keys of its
// warp's part of the slice in registers.  With the threshold bin b1 known from
// the histogram, every key at or above it (above(b1) + h[b1] keys in the row)
// is appended with its position to the row's list; after one barrier each CTA
// loads the whole list into shared memory, resolves the remaining 20 bits
// (two 10-bit digits) on it, takes its output offset from the list entries
// that lie before its slice, and emits its own candidates (kept per warp, in
// position order, in shared memory).
// Returns false, before touching anything shared, when the row does not
// qualify (the same decision in every CTA of the row): the threshold lies
// among negative scores, the list would not fit, the slices are too long for
// the registers, or the histogram does not count this row's scores.  The
// caller then runs select_row.  `cache` is laid out as for select_row;
// p.cand_cap / (NT / 32) must be at least kHistRegs * 32.
constexpr int kHistRegs = 12;
template <int NT>
__device__ bool select_row_hist(const Params &p, Shared<NT> *sh, uint32_t *cache, int row, int c, int C) {
    constexpr int NW = NT / 32;
    const int K = p.K;
    const int64_t n = (int64_t)__ldg(p.q_pos + row) + 1;
    if (n > p.Lmax || n <= K) return false;
    const int64_t chunk = ((n + C - 1) / C + 3) & ~int64_t(3);
    if (chunk > (int64_t)kHistRegs * 32 * NW || p.cand_cap / NW < kHistRegs * 32) return false;
    const int64_t lo = n < (int64_t)c * chunk ? n : (int64_t)c * chunk;
    const int64_t hi = n < lo + chunk ? n : lo + chunk;
    const int64_t len = hi - lo;
    const int warp = warp_id(), lane = lane_id();
    const uint32_t lt = (1u << lane) - 1u;
    int32_t *out = p.idx + (int64_t)row * K;
    const float *src = p.scores + (int64_t)row * p.stride;
    uint32_t *rs = p.scratch + (int64_t)row * p.scratch_row_words;
    uint32_t *ctl = rs + ctl_base(C);
    uint32_t *lkey = cache + p.cache_keys, *lpos = lkey + p.smem_list;
    const int seg = p.cand_cap / NW;
    uint32_t *wkey = lpos + p.smem_list + warp * seg, *wpos = wkey + p.cand_cap;

    // ---- the row's histogram and this thread's keys, all loads in flight together
    int64_t wlo, whi;
    warp_part<NT>(len, &wlo, &whi);
    constexpr int kHistPer = (kBins + NT - 1) / NT;
    uint32_t hv[kHistPer];
#pragma unroll
    for (int u = 0; u < kHistPer; ++u) {
        const int j = u * NT + threadIdx.x;
        hv[u] = j < kBins ? __ldcg(rs + histi_base(C, p.list_cap) + j) : 0u;
    }
    const uint32_t negatives = __ldcg(rs + histi_base(C, p.list_cap) + kBins);
    float v[kHistRegs];
#pragma unroll
    for (int i = 0; i < kHistRegs; ++i) {
        const int64_t j = wlo + i * 32 + lane;
        v[i] = j < whi ? __ldcg(src + lo + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kHistPer; ++u) {
        const int j = u * NT + threadIdx.x;
        if (j < kBins) sh->hist[j] = hv[u];
    }
    __syncthreads();
    find_threshold<NT>(sh, kBins, (uint32_t)K);
    const uint32_t b1 = (uint32_t)sh->bin;
    const uint32_t m = sh->above + sh->hist[b1];   // keys at or above bin b1 in the row
    // the histogram must count exactly this row's n scores, and the threshold
    // must lie among the non-negative ones
    if (sh->total + negatives != (uint32_t)n || sh->total < (uint32_t)K || m > (uint32_t)p.smem_list ||
        m > (uint32_t)p.list_cap)
        return false;
    uint32_t prefix = 0x80000000u | (b1 << 20), mask = 0xFFF00000u, Krem = (uint32_t)K - sh->above;
    __syncthreads();

    // ---- this warp's candidates, in position order, into its segment
    uint32_t wc = 0;
#pragma unroll
    for (int i = 0; i < kHistRegs; ++i) {
        const int64_t j = wlo + i * 32 + lane;
        const uint32_t k = float_order_key(v[i]);
        const bool cand = j < whi && k >= prefix;
        const uint32_t cm = __ballot_sync(0xffffffffu, cand);
        if (cand) {
            const uint32_t slot = wc + __popc(cm & lt);
            wkey[slot] = k;
            wpos[slot] = (uint32_t)(lo + j);
        }
        wc += __popc(cm);
    }
    if (lane == 0) sh->warp_a[warp] = wc;
    __syncwarp();
    {   // append them to the row's list, one atomic per warp
        uint32_t at = 0;
        if (lane == 0 && wc) at = atomicAdd(ctl + 4, wc);
        at = __shfl_sync(0xffffffffu, at, 0);
        uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
        for (uint32_t i = lane; i < wc; i += 32) {
            if (at + i < (uint32_t)p.list_cap) {
                gkey[at + i] = wkey[i];
                gpos[at + i] = wpos[i];
            }
        }
    }
    for (int j = threadIdx.x; j < 1024; j += NT) sh->hist[j] = 0;   // for digit 2, filled while the list loads
    if (!row_barrier<NT>(sh, ctl, (uint32_t)C, p.bar, p.status)) return true;

    // ---- the whole list into shared memory, with the digit-2 histogram of
    //      the keys in the threshold bin on the way
    {
        const uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
        for (uint32_t base = 0; base < m; base += 4 * NT) {
            uint32_t kv[4], pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t j = base + u * NT + threadIdx.x;
                kv[u] = j < m ? __ldcg(gkey + j) : 0u;
                pv[u] = j < m ? __ldcg(gpos + j) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t j = base + u * NT + threadIdx.x;
                if (j < m) {
                    lkey[j] = kv[u];
                    lpos[j] = pv[u];
                }
                warp_hist_add(sh->hist, (kv[u] >> 10) & 1023u, j < m && (kv[u] & mask) == prefix);
            }
        }
        __syncthreads();
    }
    // ---- digits 2 (histogram ready) and 3 on the list
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        const int shift = r == 0 ? 10 : 0, nb = 1024;
        if (r == 1) {
            for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = 0;
            __syncthreads();
            list_digit_hist<NT>(sh->hist, m, prefix, mask, shift, (uint32_t)nb, [&](uint32_t j, uint32_t &k) { k = lkey[j]; return true; });
            __syncthreads();
        }
        find_threshold<NT>(sh, nb, Krem);
        prefix |= (uint32_t)sh->bin << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        Krem -= sh->above;
        __syncthreads();
    }
    const uint32_t Tstar = prefix, ties = Krem;

    // ---- offset: list entries before this slice (greater in the high half, equal in the low)
    uint32_t ge = 0;
    for (uint32_t base = threadIdx.x; base < m; base += 4 * NT) {   // four entries in flight
        uint32_t k4[4], p4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool in = base + u * NT < m;
            k4[u] = in ? lkey[base + u * NT] : 0u;
            p4[u] = in ? lpos[base + u * NT] : 0xFFFFFFFFu;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if ((int64_t)p4[u] < lo) ge += k4[u] > Tstar ? 0x10000u : (k4[u] == Tstar ? 1u : 0u);
    }
    uint32_t before;
    block_scan<NT>(ge, sh->warp_tmp, &before);
    const uint32_t gt_before = before >> 16, eq_before = before & 0xFFFFu;
    const uint32_t out_pos = gt_before + (eq_before < ties ? eq_before : ties);

    // ---- emission of this CTA's candidates
    uint32_t g = 0, e = 0;
    for (uint32_t i = lane; i < wc; i += 32) {
        g += wkey[i] > Tstar;
        e += wkey[i] == Tstar;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane == 0) {
        sh->warp_b[warp] = g;
        sh->warp_c[warp] = e;
    }
    __syncthreads();
    uint32_t eq_seen = eq_before + warp_sum_prefix(sh->warp_c, warp);
    const uint32_t cta_eq = eq_before < ties ? eq_before : ties;
    uint32_t o = out_pos + warp_sum_prefix(sh->warp_b, warp) + ((eq_seen < ties ? eq_seen : ties) - cta_eq);
    if (g || (e && eq_seen < ties)) {
        for (uint32_t i0 = 0; i0 < wc; i0 += 32) {
            const uint32_t i = i0 + lane;
            const uint32_t k = i < wc ? wkey[i] : 0u;
            const bool is_eq = i < wc && k == Tstar;
            const uint32_t em = __ballot_sync(0xffffffffu, is_eq);
            const bool sel = (i < wc && k > Tstar) || (is_eq && eq_seen + __popc(em & lt) < ties);
            const uint32_t sm = __ballot_sync(0xffffffffu, sel);
            if (sel) {
                const uint32_t at = o + __popc(sm & lt);
                if (at < (uint32_t)K) out[at] = (int32_t)wpos[i];
            }
            o += __popc(sm);
            eq_seen += __popc(em);
        }
    }
    if (c == 0 && threadIdx.x == 0) p.count[row] = K;
    return true;
}

// CTA c's share of clearing row `row`'s scratch for the next call, once no
// CTA of the row reads it any more: the digit histograms, the counts and the
// list entries used, and the indexer's histogram when it was built (histi).
// The control words stay for reset_row_ctl.
// Threads tid < nt of the CTA take part.
__device__ __forceinline__ void clear_row_share(const Params &p, int row, int c, int C, bool histi, int tid, int nt) {
    uint32_t *rs = p.scratch + (int64_t)row * p.scratch_row_words;
    if (histi) {
        uint32_t *hi = rs + histi_base(C, p.list_cap);
        for (int j = c * nt + tid; j < kHistIWords; j += C * nt) hi[j] = 0;
    }
    if (C > 1) {
        for (int j = c * nt + tid; j < ctl_base(C); j += C * nt) rs[j] = 0;
        const uint32_t m2 = __ldcg(rs + ctl_base(C) + 2), m4 = __ldcg(rs + ctl_base(C) + 4);
        const uint32_t m = m2 > m4 ? m2 : m4;
        const uint32_t used = m < (uint32_t)p.list_cap ? m : (uint32_t)p.list_cap;
        uint32_t *gkey = rs + list_base(C), *gpos = gkey + p.list_cap;
        for (uint32_t j = c * nt + tid; j < used; j += C * nt) {
            gkey[j] = 0;
            gpos[j] = 0;
        }
    }
}

// Resets row `row`'s control words, once every CTA of the row has read them.
__device__ __forceinline__ void reset_row_ctl(const Params &p, int row, int C) {
    if (C > 1 && threadIdx.x < kCtlWords) p.scratch[(int64_t)row * p.scratch_row_words + ctl_base(C) + threadIdx.x] = 0;
}

}  // namespace topk
}  // namespace dsa
