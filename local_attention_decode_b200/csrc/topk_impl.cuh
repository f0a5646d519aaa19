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
// Exact radix select on the order-preserving 32-bit image of each score:
// three digit rounds (11 + 11 + 10 bits) narrow the threshold key T* and the
// number of ties at T* that still fit; one ordered compaction pass then emits,
// in increasing position order, every position with key > T* and the first
// ties positions with key == T*.  C CTAs share a row: each owns a contiguous
// slice, keeps it in shared memory when it fits, adds its non-zero histogram
// bins into the row's global histogram, and waits on a per-row counter barrier
// (bounded spin) between rounds.  Per-CTA (greater, equal) counts give each CTA
// its output offset, so the output order is a pure function of the scores.
// The row's scratch words are zeroed again before the CTAs leave.
#pragma once

#include "common.cuh"

namespace dsa {
namespace topk {

constexpr int kBins = 2048;                 // largest digit: 11 bits
constexpr int kUnroll = 8;                  // independent loads in flight per thread

// Per-row scratch (u32 words), used when C > 1 (or when the first histogram
// is produced by the indexer).
constexpr int kHist1 = 0, kHist2 = 2048, kHist3 = 4096, kCnt = 5120;
__host__ __device__ constexpr int scratch_words(int C) { return kCnt + 2 * C + 2; }   // + barrier, exit

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
    int cache_keys;
    int64_t Lmax;
};

template <int NT>
struct alignas(16) Shared {
    uint32_t hist[kBins];
    uint32_t warp_tmp[NT / 32];
    uint32_t warp_tmp2[NT / 32];
    int bin;
    uint32_t above;
    uint32_t ok;
};

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
// above(b) = number of keys in bins > b.  Result in sh->bin / sh->above.
template <int NT>
__device__ void find_threshold(Shared<NT> *sh, int nbins, uint32_t K) {
    const int per = (nbins + NT - 1) / NT;
    const int lo = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j)
        if (lo + j < nbins) mine += sh->hist[lo + j];
    uint32_t total;
    uint32_t incl = block_scan<NT>(mine, sh->warp_tmp, &total);
    uint32_t above = total - incl;      // keys in bins after this thread's range
    for (int j = per - 1; j >= 0; --j) {
        if (lo + j >= nbins) continue;
        uint32_t h = sh->hist[lo + j];
        if (above < K && K <= above + h) {
            sh->bin = lo + j;
            sh->above = above;
        }
        above += h;
    }
    __syncthreads();
}

// Barrier among the C CTAs of a row: arrive, then wait (bounded) until
// `target` arrivals have been counted.
template <int NT>
__device__ bool row_barrier(Shared<NT> *sh, uint32_t *bar, uint32_t target, uint32_t *status) {
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ok = 1;
        __threadfence();
        atomicAdd(bar, 1u);
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(bar) < target) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                flag_error(status, DSA_ERR_DEVICE_TIMEOUT);
                ok = 0;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
        sh->ok = ok;
    }
    __syncthreads();
    return sh->ok != 0;
}

// Selection of row `row` by CTA c of the C CTAs that share it.  All NT
// threads of the CTA call this.  `cache` holds p.cache_keys keys.
// hist1_ready: the row's first-digit histogram is already complete in the
// row's global scratch (built by the producer of the scores), so the first
// round reads it instead of counting.
template <int NT>
__device__ void select_row(const Params &p, Shared<NT> *sh, uint32_t *cache, int row, int c, int C,
                           bool hist1_ready) {
    const int K = p.K;
    int64_t n = (int64_t)__ldg(p.q_pos + row) + 1;
    if (n > p.Lmax) {   // a position beyond the scores buffer: flag it, select within the buffer
        if (c == 0 && threadIdx.x == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
        n = p.Lmax;
    }
    int32_t *out = p.idx + (int64_t)row * K;
    const float *src = p.scores + (int64_t)row * p.stride;
    uint32_t *rs = (C > 1 || hist1_ready) ? p.scratch + (int64_t)row * p.scratch_row_words : nullptr;

    if (n <= K) {   // every visible position is selected (same decision in all CTAs of the row)
        if (c == 0) {
            for (int j = threadIdx.x; j < K; j += NT) out[j] = j < n ? j : -1;
            if (threadIdx.x == 0) p.count[row] = (int32_t)(n > 0 ? n : 0);
        }
        if (hist1_ready) {   // the producer's histogram is not needed: clear this CTA's share
            __syncthreads();
            for (int j = c * NT + threadIdx.x; j < kHist2; j += C * NT) rs[j] = 0;
        }
        return;
    }

    const int64_t chunk = ((n + C - 1) / C + 3) & ~int64_t(3);
    const int64_t lo = n < (int64_t)c * chunk ? n : (int64_t)c * chunk;
    const int64_t hi = n < lo + chunk ? n : lo + chunk;
    const int64_t len = hi - lo;
    const bool cached = len <= p.cache_keys;

    // scores may have been written earlier in the same kernel: read them through L2 (no .nc loads)
    auto key_at = [&](int64_t j) -> uint32_t { return cached ? cache[j] : float_order_key(__ldcg(src + lo + j)); };
    // Visits keys j = base + u * NT + tid in batches of kUnroll per thread,
    // all loads of a batch issued before any is used.
    auto for_each_key = [&](auto &&fn) {
        for (int64_t base = 0; base < len; base += (int64_t)kUnroll * NT) {
            uint32_t kk[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * NT + threadIdx.x;
                kk[u] = j < len ? key_at(j) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) fn(base + u * NT + threadIdx.x, kk[u]);
        }
    };
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
        __syncthreads();
    }

    // ---- three digit rounds
    uint32_t prefix = 0, mask = 0, Krem = (uint32_t)K;
    uint32_t barrier_no = 0;
    const int shifts[3] = {21, 10, 0};
    const int nbits[3] = {11, 11, 10};
    const int hoff[3] = {kHist1, kHist2, kHist3};
    for (int r = 0; r < 3; ++r) {
        const int nb = 1 << nbits[r], sh_ = shifts[r];
        if (r == 0 && hist1_ready) {
            for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = __ldcg(rs + kHist1 + j);
            __syncthreads();
        } else {
            for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = 0;
            __syncthreads();
            // warp-aggregated increments: lanes that hit the same bin add once
            for_each_key([&](int64_t j, uint32_t k) {
                bool active = j < len && (k & mask) == prefix;
                uint32_t bin = active ? (k >> sh_) & (nb - 1) : 0xFFFFFFFFu;
                uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (active && lane_id() == __ffs(peers) - 1) atomicAdd(&sh->hist[bin], (uint32_t)__popc(peers));
            });
            __syncthreads();
            if (C > 1) {
                uint32_t *g = rs + hoff[r];
                for (int j = threadIdx.x; j < nb; j += NT)
                    if (sh->hist[j]) atomicAdd(g + j, sh->hist[j]);
                if (!row_barrier<NT>(sh, rs + kCnt + 2 * C, ++barrier_no * C, p.status)) return;
                for (int j = threadIdx.x; j < nb; j += NT) sh->hist[j] = __ldcg(g + j);
                __syncthreads();
            }
        }
        find_threshold<NT>(sh, nb, Krem);
        prefix |= (uint32_t)sh->bin << sh_;
        mask |= (uint32_t)(nb - 1) << sh_;
        Krem -= sh->above;
        __syncthreads();
    }
    const uint32_t Tstar = prefix;
    const uint32_t ties = Krem;   // how many keys equal to T* are taken (>= 1)

    // ---- per-CTA counts of keys > T* and == T*
    uint32_t gt = 0, eq = 0;
    for_each_key([&](int64_t j, uint32_t k) {
        gt += j < len && k > Tstar;
        eq += j < len && k == Tstar;
    });
    uint32_t tot_gt, tot_eq;
    block_scan<NT>(gt, sh->warp_tmp, &tot_gt);
    block_scan<NT>(eq, sh->warp_tmp, &tot_eq);
    uint32_t gt_before = 0, eq_before = 0;
    if (C > 1) {
        uint32_t *cnt = rs + kCnt;
        if (threadIdx.x == 0) {
            cnt[2 * c] = tot_gt;
            cnt[2 * c + 1] = tot_eq;
        }
        if (!row_barrier<NT>(sh, rs + kCnt + 2 * C, ++barrier_no * C, p.status)) return;
        // every CTA has read the histograms: clear this CTA's share for the next call
        for (int j = c * NT + threadIdx.x; j < kCnt; j += C * NT) rs[j] = 0;
        uint32_t a = 0, e = 0;
        for (int j = threadIdx.x; j < c; j += NT) {
            a += __ldcg(cnt + 2 * j);
            e += __ldcg(cnt + 2 * j + 1);
        }
        uint32_t t1, t2;
        block_scan<NT>(a, sh->warp_tmp, &t1);
        block_scan<NT>(e, sh->warp_tmp, &t2);
        gt_before = t1;
        eq_before = t2;
    } else if (hist1_ready) {
        __syncthreads();
        for (int j = threadIdx.x; j < kHist2; j += NT) rs[j] = 0;
    }
    const uint32_t quota = eq_before >= ties ? 0u : min(ties - eq_before, tot_eq);
    uint32_t out_pos = gt_before + min(eq_before, ties);

    // ---- ordered compaction: 4 consecutive keys per thread per step
    uint32_t eq_seen = 0;
    for (int64_t base = 0; base < len; base += 4 * NT) {
        uint32_t kk[4];
        uint32_t e_cnt = 0;
        const int64_t j0 = base + 4 * threadIdx.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            kk[u] = (j0 + u < len) ? key_at(j0 + u) : 0u;
            e_cnt += (j0 + u < len) && kk[u] == Tstar;
        }
        uint32_t e_tot;
        uint32_t e_incl = block_scan<NT>(e_cnt, sh->warp_tmp, &e_tot);
        uint32_t e_rank = eq_seen + e_incl - e_cnt;
        uint32_t sel[4], s_cnt = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            bool valid = j0 + u < len;
            bool is_eq = valid && kk[u] == Tstar;
            sel[u] = valid && (kk[u] > Tstar || (is_eq && e_rank < quota));
            e_rank += is_eq;
            s_cnt += sel[u];
        }
        uint32_t s_tot;
        uint32_t s_incl = block_scan<NT>(s_cnt, sh->warp_tmp2, &s_tot);
        uint32_t o = out_pos + s_incl - s_cnt;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (sel[u]) out[o++] = (int32_t)(lo + j0 + u);
        out_pos += s_tot;
        eq_seen += e_tot;
    }
    if (c == 0 && threadIdx.x == 0) p.count[row] = K;

    if (C > 1) {   // the last CTA of the row out clears the counts and the barrier words
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t *bar = rs + kCnt + 2 * C;
            __threadfence();
            uint32_t done = atomicAdd(bar + 1, 1u);
            if (done == (uint32_t)C - 1) {
                for (int j = 0; j < 2 * C; ++j) rs[kCnt + j] = 0;
                atomicExch(bar, 0u);
                atomicExch(bar + 1, 0u);
            }
        }
    }
}

}  // namespace topk
}  // namespace dsa
