// topk.cu -- deterministic top-k selection over indexer scores.
//
// For each query row: the min(top_k, n) positions among 0..n-1 with the
// largest scores, equal scores broken toward the lower position ("Naive-N0.5-
// Flash: no full-attention layers, and a runtime built by AI", sections "What
// 'no full-attention layers' means" -- argsort(...)[..., :index_top_k] -- and
// "How much of this did AI actually build?" -- the stable-tie argsort).
//
// Algorithm: exact radix select on the order-preserving 32-bit image of each
// score, three digit rounds (11 + 11 + 10 bits) that narrow the threshold key
// T* and the number r of ties at T* that still fit, then one ordered
// compaction pass that emits, in increasing position order, every position
// with key > T* and the first r positions with key == T*.
//
// A long row is split across C co-resident CTAs (cooperative launch).  Each
// CTA caches its contiguous slice of the row in shared memory, builds a
// shared-memory histogram per round and adds its non-zero bins into a per-row
// global histogram; a per-row counter barrier (bounded spin) separates the
// rounds.  The compaction uses per-CTA (greater, equal) counts, so the output
// order is a pure function of the scores: run-to-run bit-identical.
// The per-row scratch is zeroed again by the CTAs before they exit.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace topk {

constexpr int kThreads = 512;
constexpr int kBins = 2048;                 // largest digit: 11 bits
constexpr int kMinChunk = 4096;             // keys per CTA below which a row is not split further
constexpr int kMaxCacheKeys = 40 * 1024;    // 160 KB of cached keys per CTA
constexpr int kUnroll = 8;                  // independent loads in flight per thread

// Per-row scratch (u32 words), used only when C > 1.
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

struct alignas(16) Shared {
    uint32_t hist[kBins];
    uint32_t warp_tmp[kThreads / 32];
    uint32_t warp_tmp2[kThreads / 32];
    int bin;
    uint32_t above;
    uint32_t ok;
};

// Inclusive block scan of one value per thread; returns the inclusive prefix
// and writes the block total to *total.
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t *warp_tmp, uint32_t *total) {
    const int lane = lane_id(), warp = warp_id();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < kThreads / 32 ? warp_tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < kThreads / 32) warp_tmp[lane] = w;
    }
    __syncthreads();
    uint32_t add = warp > 0 ? warp_tmp[warp - 1] : 0;
    *total = warp_tmp[kThreads / 32 - 1];
    __syncthreads();
    return v + add;
}

// Threshold bin of a histogram: the bin b with above(b) < K <= above(b) + h[b],
// above(b) = number of keys in bins > b.  Result in sh->bin / sh->above.
__device__ void find_threshold(Shared *sh, int nbins, uint32_t K) {
    const int per = nbins / kThreads;   // 4 or 2 bins per thread
    const int lo = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j) mine += sh->hist[lo + j];
    uint32_t total;
    uint32_t incl = block_scan(mine, sh->warp_tmp, &total);
    uint32_t above = total - incl;      // keys in bins after this thread's range
    for (int j = per - 1; j >= 0; --j) {
        uint32_t h = sh->hist[lo + j];
        if (above < K && K <= above + h) {
            sh->bin = lo + j;
            sh->above = above;
        }
        above += h;
    }
    __syncthreads();
}

// Per-row barrier across the C CTAs of a row; bounded spin.
__device__ bool row_barrier(Shared *sh, uint32_t *bar, uint32_t target, uint32_t *status) {
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

__global__ void __launch_bounds__(kThreads)
topk_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Shared *sh = reinterpret_cast<Shared *>(smem_raw);
    uint32_t *cache = reinterpret_cast<uint32_t *>(smem_raw + sizeof(Shared));

    const int row = blockIdx.x / p.C, c = blockIdx.x % p.C, C = p.C;
    const int K = p.K;
    int64_t n = (int64_t)__ldg(p.q_pos + row) + 1;
    if (n > p.Lmax) {   // a position beyond the scores buffer: flag it, select within the buffer
        if (c == 0 && threadIdx.x == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
        n = p.Lmax;
    }
    int32_t *out = p.idx + (int64_t)row * K;
    const float *src = p.scores + (int64_t)row * p.stride;

    if (n <= K) {   // every visible position is selected (same decision in all CTAs of the row)
        if (c == 0) {
            for (int j = threadIdx.x; j < K; j += kThreads) out[j] = j < n ? j : -1;
            if (threadIdx.x == 0) p.count[row] = (int32_t)(n > 0 ? n : 0);
        }
        return;
    }

    const int64_t chunk = ((n + C - 1) / C + 3) & ~int64_t(3);
    const int64_t lo = n < (int64_t)c * chunk ? n : (int64_t)c * chunk;
    const int64_t hi = n < lo + chunk ? n : lo + chunk;
    const int64_t len = hi - lo;
    const bool cached = len <= p.cache_keys;
    uint32_t *rs = C > 1 ? p.scratch + (int64_t)row * p.scratch_row_words : nullptr;

    auto key_at = [&](int64_t j) -> uint32_t { return cached ? cache[j] : float_order_key(__ldg(src + lo + j)); };
    // Visits keys j = base + u * kThreads + tid in batches of kUnroll per
    // thread, all loads of a batch issued before any is used.
    auto for_each_key = [&](auto &&fn) {
        for (int64_t base = 0; base < len; base += (int64_t)kUnroll * kThreads) {
            uint32_t kk[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * kThreads + threadIdx.x;
                kk[u] = j < len ? key_at(j) : 0u;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) fn(base + u * kThreads + threadIdx.x, kk[u]);
        }
    };
    if (cached) {
        for (int64_t base = 0; base < len; base += (int64_t)kUnroll * kThreads) {
            float v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * kThreads + threadIdx.x;
                v[u] = j < len ? __ldg(src + lo + j) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t j = base + u * kThreads + threadIdx.x;
                if (j < len) cache[j] = float_order_key(v[u]);
            }
        }
        __syncthreads();
    }

    // ---- three digit rounds
    uint32_t prefix = 0, mask = 0, Krem = (uint32_t)K;
    const int shifts[3] = {21, 10, 0};
    const int nbits[3] = {11, 11, 10};
    const int hoff[3] = {kHist1, kHist2, kHist3};
    for (int r = 0; r < 3; ++r) {
        const int nb = 1 << nbits[r], sh_ = shifts[r];
        for (int j = threadIdx.x; j < nb; j += kThreads) sh->hist[j] = 0;
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
            for (int j = threadIdx.x; j < nb; j += kThreads)
                if (sh->hist[j]) atomicAdd(g + j, sh->hist[j]);
            if (!row_barrier(sh, rs + kCnt + 2 * C, (uint32_t)(r + 1) * C, p.status)) return;
            for (int j = threadIdx.x; j < nb; j += kThreads) sh->hist[j] = __ldcg(g + j);
            __syncthreads();
        }
        find_threshold(sh, nb, Krem);
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
    block_scan(gt, sh->warp_tmp, &tot_gt);
    block_scan(eq, sh->warp_tmp, &tot_eq);
    uint32_t gt_before = 0, eq_before = 0;
    if (C > 1) {
        uint32_t *cnt = rs + kCnt;
        if (threadIdx.x == 0) {
            cnt[2 * c] = tot_gt;
            cnt[2 * c + 1] = tot_eq;
        }
        if (!row_barrier(sh, rs + kCnt + 2 * C, 4u * C, p.status)) return;
        // every CTA has read the histograms: clear this CTA's share for the next call
        for (int j = c * kThreads + threadIdx.x; j < kCnt; j += C * kThreads) rs[j] = 0;
        uint32_t a = 0, e = 0;
        for (int j = threadIdx.x; j < c; j += kThreads) {
            a += __ldcg(cnt + 2 * j);
            e += __ldcg(cnt + 2 * j + 1);
        }
        uint32_t t1, t2;
        block_scan(a, sh->warp_tmp, &t1);
        block_scan(e, sh->warp_tmp, &t2);
        gt_before = t1;
        eq_before = t2;
    }
    const uint32_t quota = eq_before >= ties ? 0u : min(ties - eq_before, tot_eq);
    uint32_t out_pos = gt_before + min(eq_before, ties);

    // ---- ordered compaction: 4 consecutive keys per thread per step
    uint32_t eq_seen = 0;
    for (int64_t base = 0; base < len; base += 4 * kThreads) {
        uint32_t kk[4];
        uint32_t e_cnt = 0;
        const int64_t j0 = base + 4 * threadIdx.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            kk[u] = (j0 + u < len) ? key_at(j0 + u) : 0u;
            e_cnt += (j0 + u < len) && kk[u] == Tstar;
        }
        uint32_t e_tot;
        uint32_t e_incl = block_scan(e_cnt, sh->warp_tmp, &e_tot);
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
        uint32_t s_incl = block_scan(s_cnt, sh->warp_tmp2, &s_tot);
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

int plan_topk(int B, int T, int64_t Lmax, int top_k, TopkPlan *plan) {
    using namespace topk;
    const DeviceInfo &dev = device_info();
    plan->rows = B * T;
    plan->threads = kThreads;
    plan->Lmax = Lmax;
    int C = 1;
    if (dev.num_sms > 0 && Lmax > top_k) {
        int co_resident = dev.num_sms;   // one CTA per SM is always co-resident at this size
        C = (int)std::max<int64_t>(1, std::min<int64_t>(co_resident / std::max(1, plan->rows),
                                                       (Lmax + kMinChunk - 1) / kMinChunk));
    }
    int64_t chunk = ((Lmax + C - 1) / C + 3) & ~int64_t(3);
    plan->ctas_per_row = C;
    plan->cache_keys = (int)std::min<int64_t>(chunk, kMaxCacheKeys);
    plan->smem = sizeof(Shared) + (size_t)plan->cache_keys * 4;
    plan->scratch_bytes = C > 1 ? (size_t)plan->rows * scratch_words(C) * 4 : 0;
    return DSA_OK;
}

int launch_topk(const TopkPlan &plan, const float *scores, int64_t stride, const int32_t *q_pos, int top_k,
                int32_t *idx, int32_t *count, uint32_t *scratch, uint32_t *status, cudaStream_t stream) {
    using namespace topk;
    Params p;
    p.scores = scores;
    p.stride = stride;
    p.q_pos = q_pos;
    p.rows = plan.rows;
    p.K = top_k;
    p.C = plan.ctas_per_row;
    p.idx = idx;
    p.count = count;
    p.scratch = scratch;
    p.scratch_row_words = scratch_words(plan.ctas_per_row);
    p.status = status;
    p.cache_keys = plan.cache_keys;
    p.Lmax = plan.Lmax;
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(topk)");
    const unsigned grid = (unsigned)(plan.rows * plan.ctas_per_row);
    if (plan.ctas_per_row > 1) {
        // the CTAs of a row wait on one another: they must all be resident
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = plan.smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, topk_kernel, p);
    } else {
        topk_kernel<<<grid, kThreads, plan.smem, stream>>>(p);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return cuda_fail(e, "topk launch");
    return DSA_OK;
}

}  // namespace dsa
