// shard.cu -- the pieces of a DSA decode layer-step whose context is split
// across ranks (one contiguous slice of positions per rank):
//   candidates  the rank's local selection (its indexer scores and top-k over
//               its slice) turned into (score, global position) pairs;
//   merge       from every rank's pairs, the global top-k (score descending,
//               ties to the lower position -- the same rule as the one-GPU
//               selection) in position order, and this rank's share of it as
//               local positions;
//   combine     the ranks' attention outputs over their shares (each without
//               the sink) merged by their log-sum-exp, the sink added once.
// The exchanges between the steps are the caller's collectives.  Together
// with dsa_indexer_scores, dsa_topk_select and sparse_gqa_attn_decode on each
// rank's slice they compute the layer-step of "Naive-N0.5-Flash: no
// full-attention layers, and a runtime built by AI" ("Inside a DSA layer":
// score every visible key, keep the top 2,048, attend to those) exactly as on
// one GPU: the selected set is the same, and the attention is the same sum
// split by owner.
#include "common.cuh"
#include "kernels.h"
#include "topk_impl.cuh"

namespace dsa {
namespace shard {

constexpr int kThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------- candidates
// One thread per (row, j): idx from the local selection (local positions,
// -1 padded) -> (score at it, global position) or (-inf, -1).
__global__ void candidates_kernel(const float *scores, int64_t stride, const int32_t *idx, int K, int rows,
                                  int64_t offset, float *cand_score, int32_t *cand_pos) {
    pdl_begin();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)rows * K) return;
    const int r = (int)(i / K);
    const int32_t l = __ldg(idx + i);
    if (l >= 0) {
        cand_score[i] = __ldg(scores + (int64_t)r * stride + l);
        cand_pos[i] = (int32_t)(offset + l);
    } else {
        cand_score[i] = -INFINITY;
        cand_pos[i] = -1;
    }
}

// ---------------------------------------------------------------- merge
// One CTA per row: the n = N * K pairs in shared memory in rank order (each
// rank's slice precedes the next one's, and each rank's pairs are in position
// order, so the valid pairs are in position order), the k-th largest order
// key by an exact 11 + 11 + 10-bit radix select, then every pair above it and
// the first `ties` pairs equal to it (the lower positions) compacted in
// position order.  Pairs with position -1 are never selected.
__global__ void __launch_bounds__(kThreads)
merge_kernel(const float *cand_score, const int32_t *cand_pos, int N, int K, int rows, int64_t rank_offset,
             int64_t rank_len, int32_t *idx_out, int32_t *count_out, int32_t *local_idx, int32_t *local_count) {
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_begin();
    const int r = blockIdx.x, t = threadIdx.x, n = N * K;
    auto *sh = reinterpret_cast<topk::Shared<kThreads> *>(smem);
    uint32_t *key = reinterpret_cast<uint32_t *>(smem + ((sizeof(topk::Shared<kThreads>) + 15) & ~size_t(15)));
    int32_t *pos = reinterpret_cast<int32_t *>(key + n);
    uint32_t valid = 0;
    for (int i = t; i < n; i += kThreads) {
        const int rk = i / K, j = i % K;
        const int64_t src = ((int64_t)rk * rows + r) * K + j;
        const int32_t p = __ldg(cand_pos + src);
        pos[i] = p;
        key[i] = p >= 0 ? float_order_key(__ldg(cand_score + src)) : 0u;
        valid += p >= 0;
    }
    uint32_t m;
    topk::block_scan<kThreads>(valid, sh->warp_tmp, &m);
    const uint32_t kk = m < (uint32_t)K ? m : (uint32_t)K;
    uint32_t prefix = 0, mask = 0, Krem = kk;
    if (kk > 0) {
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0), nb = pass == 2 ? 1024 : 2048;
            for (int b = t; b < nb; b += kThreads) sh->hist[b] = 0;
            __syncthreads();
            list_digit_hist<kThreads>(sh->hist, (uint32_t)n, prefix, mask, shift, (uint32_t)nb,
                                      [&](uint32_t i, uint32_t &k) {
                                          k = key[i];
                                          return pos[i] >= 0;
                                      });
            __syncthreads();
            topk::find_threshold<kThreads>(sh, nb, Krem);
            prefix |= (uint32_t)sh->bin << shift;
            mask |= (uint32_t)(nb - 1) << shift;
            Krem -= sh->above;
            __syncthreads();
        }
    }
    const uint32_t Tstar = prefix, ties = Krem;
    const int per = (n + kThreads - 1) / kThreads;
    const int lo = min(n, t * per), hi = min(n, lo + per);
    uint32_t g = 0, e = 0;
    if (kk > 0)
        for (int i = lo; i < hi; ++i) {
            if (pos[i] < 0) continue;
            g += key[i] > Tstar;
            e += key[i] == Tstar;
        }
    const uint32_t packed = (g << 16) | e;
    uint32_t dummy;
    const uint32_t excl = topk::block_scan<kThreads>(packed, sh->warp_tmp, &dummy) - packed;
    uint32_t gb = excl >> 16, eb = excl & 0xFFFFu;
    int32_t *out = idx_out + (int64_t)r * K;
    if (kk > 0)
        for (int i = lo; i < hi; ++i) {
            if (pos[i] < 0) continue;
            if (key[i] > Tstar) {
                out[gb + (eb < ties ? eb : ties)] = pos[i];
                ++gb;
            } else if (key[i] == Tstar) {
                if (eb < ties) out[gb + eb] = pos[i];
                ++eb;
            }
        }
    for (int j = (int)kk + t; j < K; j += kThreads) out[j] = -1;
    if (t == 0) count_out[r] = (int32_t)kk;
    __syncthreads();
    // this rank's share, as local positions, compacted in order (one warp)
    if (local_idx && t < 32) {
        int32_t *lout = local_idx + (int64_t)r * K;
        uint32_t c = 0;
        for (int j0 = 0; j0 < (int)kk; j0 += 32) {
            const int j = j0 + t;
            const int32_t p = j < (int)kk ? __ldcg(out + j) : -1;
            const bool mine = p >= 0 && p >= rank_offset && p < rank_offset + rank_len;
            const uint32_t bm = __ballot_sync(0xffffffffu, mine);
            if (mine) lout[c + __popc(bm & ((1u << t) - 1u))] = (int32_t)(p - rank_offset);
            c += __popc(bm);
        }
        for (uint32_t j = c + t; j < (uint32_t)K; j += 32) lout[j] = -1;
        if (t == 0) local_count[r] = (int32_t)c;
    }
}

// ------------------------------------------------------------ positions
// q_pos_local = min(q_pos - offset, len - 1): the last position of the slice
// a query sees (every query is at or after the slice's start).
__global__ void positions_kernel(const int32_t *q_pos, int rows, int64_t offset, int64_t len, int32_t *q_local,
                                 uint32_t *bad) {
    pdl_begin();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows) return;
    const int64_t p = (int64_t)__ldg(q_pos + i) - offset;
    if (p < 0) atomicOr(bad, 1u);
    q_local[i] = (int32_t)(p < 0 ? 0 : (p < len ? p : len - 1));
}

// -------------------------------------------------------------- combine
// One CTA of 128 threads per (row, head): thread d takes column d of the
// head's output.  Each rank's O_r is normalised over its share; with
// lse_r = ln sum over the share of e^{s}, the full output is
// sum_r e^{lse_r - LSE} O_r, LSE = ln(sum_r e^{lse_r} + e^{sink}).
__global__ void __launch_bounds__(128)
combine_kernel(const __nv_bfloat16 *O_all, const float *lse_all, int N, int64_t rows_heads, const float *sink,
               __nv_bfloat16 *O, float *lse) {
    pdl_begin();
    const int64_t gw = blockIdx.x;
    const int d = threadIdx.x, h = (int)(gw % DSA_Q_HEADS);
    float M = sink ? __ldg(sink + h) * kLog2e : -INFINITY;
    for (int r = 0; r < N; ++r) M = fmaxf(M, __ldg(lse_all + r * rows_heads + gw) * kLog2e);
    float acc = 0.f, den = (sink && M != -INFINITY) ? exp2f(__ldg(sink + h) * kLog2e - M) : 0.f;
    for (int r = 0; r < N; ++r) {
        const float l = __ldg(lse_all + r * rows_heads + gw) * kLog2e;
        if (l == -INFINITY) continue;
        const float w = exp2f(l - M);
        acc += w * __bfloat162float(O_all[(r * rows_heads + gw) * DSA_V_DIM + d]);
        den += w;
    }
    O[gw * DSA_V_DIM + d] = __float2bfloat16_rn(den > 0.f ? acc / den : 0.f);
    if (lse && d == 0) lse[gw] = den > 0.f ? (M + log2f(den)) / kLog2e : -INFINITY;
}

}  // namespace shard

int launch_shard_candidates(const float *scores, int64_t stride, const int32_t *idx, int K, int rows, int64_t offset,
                            float *cand_score, int32_t *cand_pos, cudaStream_t stream) {
    const int64_t n = (int64_t)rows * K;
    cudaError_t e = launch_kernel(shard::candidates_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream,
                                  scores, stride, idx, K, rows, offset, cand_score, cand_pos);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "shard candidates launch");
}

int launch_shard_merge(const float *cand_score, const int32_t *cand_pos, int N, int K, int rows, int64_t rank_offset,
                       int64_t rank_len, int32_t *idx_out, int32_t *count_out, int32_t *local_idx,
                       int32_t *local_count, cudaStream_t stream) {
    const size_t smem = ((sizeof(topk::Shared<shard::kThreads>) + 15) & ~size_t(15)) + (size_t)N * K * 8;
    if (int rc = ensure_smem_limit((const void *)shard::merge_kernel, smem, "cudaFuncSetAttribute(shard merge)")) return rc;
    cudaError_t e = launch_kernel(shard::merge_kernel, dim3(rows), dim3(shard::kThreads), smem, stream, cand_score,
                                  cand_pos, N, K, rows, rank_offset, rank_len, idx_out, count_out, local_idx,
                                  local_count);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "shard merge launch");
}

int launch_shard_positions(const int32_t *q_pos, int rows, int64_t offset, int64_t len, int32_t *q_local,
                           uint32_t *bad, cudaStream_t stream) {
    cudaError_t e = launch_kernel(shard::positions_kernel, dim3((rows + 127) / 128), dim3(128), 0, stream, q_pos, rows,
                                  offset, len, q_local, bad);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "shard positions launch");
}

int launch_shard_combine(const __nv_bfloat16 *O_all, const float *lse_all, int N, int rows, const float *sink,
                         __nv_bfloat16 *O, float *lse, cudaStream_t stream) {
    const int64_t rh = (int64_t)rows * DSA_Q_HEADS;
    cudaError_t e = launch_kernel(shard::combine_kernel, dim3((unsigned)rh), dim3(128), 0, stream, O_all, lse_all, N,
                                  rh, sink, O, lse);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "shard combine launch");
}

}  // namespace dsa
