// kl.cu -- the indexer warm-up target: for each query token, the average over
// the 64 heads of each head's dense softmax attention over the visible keys
// (no sink), and the KL divergence from it to the softmax of the indexer
// scores.  ("Naive-N0.5-Flash: no full-attention layers, and a runtime built
// by AI", section "Inside a DSA layer: the lightning indexer": the indexer is
// first trained alone, aligned to a full-attention reference by a KL
// objective; "2,122 tok/s, Zero Full-Attention Layers", section "What's
// genuinely new": the converted layers keep full attention during the warm-up
// and supervise the indexer through a KL-divergence loss.)
//
//   P[s] = (1/64) sum_h softmax_s(sm_scale Q[h] . K[s][h / (64 / G)])
//   KL   = sum_s P[s] (ln P[s] - ln softmax_s(I)[s]),   s = 0 .. q_pos
//
// Four kernels, all reductions in a fixed order (the results are the same run
// to run):
//   stats   per (token, KV head, 64-key chunk): the group's 64/G x 64 logits
//           on the tensor cores (mma.sync bf16, fp32 accumulation), each
//           head's chunk max and sum of exponentials; per (token, chunk) the
//           same for the indexer scores;
//   totals  per (token, head) and per token for the indexer: the log-sum-exp
//           over the chunks;
//   target  per (token, chunk): the logits again, P for each key (written out
//           if asked) and the chunk's share of the KL;
//   final   per token: the KL.
#include <cmath>

#include "attention_impl.cuh"

namespace dsa {
namespace kl {

using attn::kLog2e;
using attn::kQS;
constexpr int kChunk = 64;
constexpr int kTeam = 128;
constexpr int kMaxTeams = 4;

struct Params {
    const __nv_bfloat16 *Q;     // [BT][64][192]
    const __nv_bfloat16 *K;     // [rows][G][192]
    int G;
    const int32_t *block_table;
    int32_t max_pages, page_size;
    int64_t seq_stride, num_rows;
    const float *scores;        // [BT][stride]
    int64_t scores_stride;
    const int32_t *q_pos;       // [BT]
    int T;
    int64_t Lmax;
    int chunks;
    float scale_log2;
    float2 *stats;              // [BT][64][chunks]  (max, sum) in the log2 domain
    float2 *stats_i;            // [BT][chunks]
    float2 *tot;                // [BT][65]
    float *kl_part;             // [BT][chunks]
    float *kl_out;              // [BT]
    float *target;              // [BT][target_stride] or null
    int64_t target_stride;
    uint32_t *status;
};

struct TeamSmem {
    __nv_bfloat16 q[16 * kQS];
    __nv_bfloat16 k[kChunk * kQS];
    int64_t row[kChunk];
    float red_m[4][16];
    float red_l[4][16];
};

__device__ __forceinline__ int64_t visible_keys(const Params &p, int bt) {
    int64_t n = (int64_t)__ldg(p.q_pos + bt) + 1;
    if (n > p.Lmax) n = p.Lmax;
    return n < 0 ? 0 : n;
}

__device__ __forceinline__ bool key_row(const Params &p, int b, int64_t pos, int64_t *row) {
    if (p.block_table == nullptr) {
        if (pos >= p.seq_stride) return false;
        *row = (int64_t)b * p.seq_stride + pos;
    } else {
        const int64_t page = pos / p.page_size;
        if (page >= p.max_pages) return false;
        const int32_t id = __ldg(p.block_table + (int64_t)b * p.max_pages + page);
        if (id < 0) return false;
        *row = (int64_t)id * p.page_size + pos % p.page_size;
    }
    return *row < p.num_rows;
}

// The logits (log2 domain, -inf for a key that is not visible) of the heads
// of KV group g against the keys [c*64, c*64+64) of token bt, by one team
// (tid 0..127, named barrier `bar`): warp w holds keys w*16 .. w*16+15,
// rows lane/4 and lane/4 + 8, in the mma.sync accumulator layout s[2][4].
__device__ __forceinline__ void team_logits(const Params &p, TeamSmem &sm, int bt, int g, int c, int64_t n, int tid,
                                            int bar, float (&s)[2][4]) {
    const int hpg = DSA_Q_HEADS / p.G, warp = tid >> 5, lane = tid & 31;
    const int b = bt / p.T;
    const int64_t k0 = (int64_t)c * kChunk;
    if (tid < kChunk) {
        int64_t row = -1;
        const int64_t pos = k0 + tid;
        if (pos < n && !key_row(p, b, pos, &row)) {
            flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
            row = -1;
        }
        sm.row[tid] = pos < n ? row : -1;
    }
    const __nv_bfloat16 *qg = p.Q + ((int64_t)bt * DSA_Q_HEADS + g * hpg) * DSA_QK_DIM;
    for (int i = tid; i < 16 * (DSA_QK_DIM / 8); i += kTeam) {
        const int r = i / (DSA_QK_DIM / 8), col = (i % (DSA_QK_DIM / 8)) * 8;
        __nv_bfloat16 *dst = sm.q + r * kQS + col;
        if (r < hpg) attn::cp_async16(dst, qg + (int64_t)r * DSA_QK_DIM + col);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    attn::team_sync(bar);
    for (int i = tid; i < kChunk * (DSA_QK_DIM / 8); i += kTeam) {
        const int r = i / (DSA_QK_DIM / 8), col = (i % (DSA_QK_DIM / 8)) * 8;
        __nv_bfloat16 *dst = sm.k + r * kQS + col;
        const int64_t row = sm.row[r];
        if (row >= 0) attn::cp_async16(dst, p.K + (row * p.G + g) * DSA_QK_DIM + col);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    attn::cp_async_commit();
    attn::cp_async_wait_all();
    attn::team_sync(bar);
    const int key0 = warp * 16;
#pragma unroll
    for (int a = 0; a < 2; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
    const uint32_t q_base = smem_u32(sm.q), k_base = smem_u32(sm.k);
#pragma unroll
    for (int kk = 0; kk < DSA_QK_DIM / 16; ++kk) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        attn::ldsm_x4(q_base + ((lane & 15) * kQS + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
        attn::ldsm_x4(k_base + ((key0 + (lane >> 4) * 8 + (lane & 7)) * kQS + kk * 16 + ((lane >> 3) & 1) * 8) * 2,
                      b0, b1, b2, b3);
        attn::mma_bf16(s[0], a0, a1, a2, a3, b0, b1);
        attn::mma_bf16(s[1], a0, a1, a2, a3, b2, b3);
    }
    const int cq = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = key0 + nt * 8 + cq * 2 + (e & 1);
            s[nt][e] = sm.row[key] >= 0 ? s[nt][e] * p.scale_log2 : -INFINITY;
        }
}

// ---------------------------------------------------------------- stats
__global__ void __launch_bounds__(kTeam)
kl_stats_kernel(const Params p) {
    __shared__ TeamSmem sm;
    pdl_begin();
    const int c = blockIdx.x, g = blockIdx.y, bt = blockIdx.z, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, g0 = lane >> 2;
    const int hpg = DSA_Q_HEADS / p.G;
    const int64_t n = visible_keys(p, bt);
    if (g == 0 && tid < 32) {   // the indexer scores of the chunk
        float m = -INFINITY;
        float v[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t s = (int64_t)c * kChunk + u * 32 + tid;
            v[u] = s < n ? __ldg(p.scores + (int64_t)bt * p.scores_stride + s) * kLog2e : -INFINITY;
            m = fmaxf(m, v[u]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
#pragma unroll
        for (int u = 0; u < 2; ++u) l += m == -INFINITY ? 0.f : exp2f(v[u] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (tid == 0) p.stats_i[(int64_t)bt * p.chunks + c] = make_float2(m, l);
    }
    if ((int64_t)c * kChunk >= n) {   // nothing visible in this chunk
        if (tid < hpg) p.stats[((int64_t)bt * DSA_Q_HEADS + g * hpg + tid) * p.chunks + c] = make_float2(-INFINITY, 0.f);
        return;
    }
    float s[2][4];
    team_logits(p, sm, bt, g, c, n, tid, 1, s);
    // per head row: the chunk max, then the sum of exponentials below it
    float mr[2] = {fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1])),
                   fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]))};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        mr[r] = fmaxf(mr[r], __shfl_xor_sync(0xffffffffu, mr[r], 1));
        mr[r] = fmaxf(mr[r], __shfl_xor_sync(0xffffffffu, mr[r], 2));
    }
    if ((lane & 3) == 0) {
        sm.red_m[warp][g0] = mr[0];
        sm.red_m[warp][g0 + 8] = mr[1];
    }
    __syncthreads();
    float M[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = g0 + 8 * r;
        M[r] = fmaxf(fmaxf(sm.red_m[0][row], sm.red_m[1][row]), fmaxf(sm.red_m[2][row], sm.red_m[3][row]));
    }
    float lr[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) lr[e >> 1] += M[e >> 1] == -INFINITY ? 0.f : exp2f(s[nt][e] - M[e >> 1]);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 1);
        lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 2);
    }
    if ((lane & 3) == 0) {
        sm.red_l[warp][g0] = lr[0];
        sm.red_l[warp][g0 + 8] = lr[1];
    }
    __syncthreads();
    if (tid < hpg) {
        const float m = fmaxf(fmaxf(sm.red_m[0][tid], sm.red_m[1][tid]), fmaxf(sm.red_m[2][tid], sm.red_m[3][tid]));
        const float l = (sm.red_l[0][tid] + sm.red_l[1][tid]) + (sm.red_l[2][tid] + sm.red_l[3][tid]);
        p.stats[((int64_t)bt * DSA_Q_HEADS + g * hpg + tid) * p.chunks + c] = make_float2(m, l);
    }
}

// --------------------------------------------------------------- totals
// One block per token: thread h < 64 the head's log-sum-exp over the chunks
// (max first, then the rescaled sums, chunks in order); thread 64 the same
// for the indexer scores.
__global__ void __launch_bounds__(96)
kl_totals_kernel(const Params p) {
    pdl_begin();
    const int bt = blockIdx.x, h = threadIdx.x;
    if (h > DSA_Q_HEADS) return;
    const float2 *st = h < DSA_Q_HEADS ? p.stats + ((int64_t)bt * DSA_Q_HEADS + h) * p.chunks
                                       : p.stats_i + (int64_t)bt * p.chunks;
    float M = -INFINITY;
    for (int c = 0; c < p.chunks; ++c) M = fmaxf(M, __ldg(&st[c].x));
    float L = 0.f;
    for (int c = 0; c < p.chunks; ++c) {
        const float2 v = __ldg(st + c);
        if (v.x != -INFINITY) L += v.y * exp2f(v.x - M);
    }
    p.tot[(int64_t)bt * (DSA_Q_HEADS + 1) + h] = make_float2(M, L);
}

// --------------------------------------------------------------- target
// One block per (chunk, token), min(G, 4) teams; team t takes the KV groups
// t, t + 4, ...; P of each key summed over the heads in shared memory (groups
// in order), then thread j < 64 takes key j.
__global__ void __launch_bounds__(kMaxTeams * kTeam)
kl_target_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    pdl_begin();
    const int c = blockIdx.x, bt = blockIdx.y, tid = threadIdx.x;
    const int team = tid / kTeam, ttid = tid % kTeam, lane = tid & 31, g0 = lane >> 2, cq = lane & 3;
    const int warp = ttid >> 5;
    const int teams = p.G < kMaxTeams ? p.G : kMaxTeams, hpg = DSA_Q_HEADS / p.G;
    TeamSmem &sm = reinterpret_cast<TeamSmem *>(smem_raw)[team];
    float *gsum = reinterpret_cast<float *>(smem_raw + kMaxTeams * sizeof(TeamSmem));   // [G][64]
    const int64_t n = visible_keys(p, bt);
    const int64_t k0 = (int64_t)c * kChunk;
    if (k0 >= n) return;   // the whole block: no key of this chunk is visible
    const float2 *tot = p.tot + (int64_t)bt * (DSA_Q_HEADS + 1);
    for (int g = team; g < p.G; g += teams) {
        float s[2][4];
        team_logits(p, sm, bt, g, c, n, ttid, 1 + team, s);
        // each row's exp2(s - M_h) / L_h, summed over the group's heads per key
        float e[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int row = g0 + 8 * r;
            const float2 t = row < hpg ? tot[g * hpg + row] : make_float2(-INFINITY, 0.f);
            const float inv = t.y > 0.f ? 1.0f / t.y : 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                e[nt][2 * r] = (row < hpg && t.x != -INFINITY) ? exp2f(s[nt][2 * r] - t.x) * inv : 0.f;
                e[nt][2 * r + 1] = (row < hpg && t.x != -INFINITY) ? exp2f(s[nt][2 * r + 1] - t.x) * inv : 0.f;
            }
        }
        // sum over the 16 rows of the accumulator: rows g0 and g0 + 8 in this lane, g0 over lanes (xor 4, 8, 16)
        float colsum[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float v = e[nt][u] + e[nt][2 + u];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                colsum[nt][u] = v;
            }
        if (g0 == 0) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int u = 0; u < 2; ++u) gsum[g * kChunk + warp * 16 + nt * 8 + cq * 2 + u] = colsum[nt][u];
        }
        attn::team_sync(1 + team);
    }
    __syncthreads();
    if (tid < kChunk) {
        const int64_t s = k0 + tid;
        float term = 0.f;
        if (s < n) {
            float P = 0.f;
            for (int g = 0; g < p.G; ++g) P += gsum[g * kChunk + tid];
            P *= 1.0f / DSA_Q_HEADS;
            const float2 ti = tot[DSA_Q_HEADS];
            const float lse_i = (ti.x + log2f(ti.y)) / kLog2e;   // natural log-sum-exp of the indexer scores
            const float I = __ldg(p.scores + (int64_t)bt * p.scores_stride + s);
            if (P > 0.f) term = P * (logf(P) - (I - lse_i));
            if (p.target) p.target[(int64_t)bt * p.target_stride + s] = P;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
        if (lane == 0) sm.red_m[0][tid >> 5] = term;   // two warps
    }
    __syncthreads();
    if (tid == 0) p.kl_part[(int64_t)bt * p.chunks + c] = sm.red_m[0][0] + sm.red_m[0][1];
}

// ---------------------------------------------------------------- final
// One warp per token: the chunk terms, lanes strided, then a fixed tree.
__global__ void __launch_bounds__(32)
kl_final_kernel(const Params p) {
    pdl_begin();
    const int bt = blockIdx.x, lane = threadIdx.x;
    const int64_t n = visible_keys(p, bt);
    const int used = (int)((n + kChunk - 1) / kChunk);
    float v = 0.f;
    for (int c = lane; c < used; c += 32) v += p.kl_part[(int64_t)bt * p.chunks + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) p.kl_out[bt] = v;
}

}  // namespace kl

size_t kl_workspace_bytes(int B, int T, int64_t Lmax) {
    const int64_t chunks = (Lmax + kl::kChunk - 1) / kl::kChunk;
    const size_t bt = (size_t)B * T;
    return bt * DSA_Q_HEADS * chunks * 8 + bt * chunks * 8 + bt * (DSA_Q_HEADS + 1) * 8 + bt * chunks * 4 + 1024;
}

int launch_indexer_kl(const KlArgs &a, cudaStream_t stream) {
    using namespace kl;
    const dsa_kv_t *kv = a.kv;
    Params p;
    p.Q = a.Q;
    p.K = reinterpret_cast<const __nv_bfloat16 *>(kv->k);
    p.G = kv->num_kv_heads;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages;
    p.page_size = kv->page_size;
    p.seq_stride = kv->seq_stride;
    p.num_rows = kv->num_rows;
    p.scores = a.scores;
    p.scores_stride = a.scores_stride;
    p.q_pos = a.q_pos;
    p.T = a.T;
    p.Lmax = a.Lmax;
    p.chunks = (int)((a.Lmax + kChunk - 1) / kChunk);
    p.scale_log2 = a.sm_scale * kLog2e;
    const size_t bt = (size_t)a.B * a.T;
    uint8_t *w = static_cast<uint8_t *>(a.scratch);
    p.stats = reinterpret_cast<float2 *>(w);
    w += bt * DSA_Q_HEADS * p.chunks * 8;
    p.stats_i = reinterpret_cast<float2 *>(w);
    w += bt * p.chunks * 8;
    p.tot = reinterpret_cast<float2 *>(w);
    w += bt * (DSA_Q_HEADS + 1) * 8;
    p.kl_part = reinterpret_cast<float *>(w);
    p.kl_out = a.kl_out;
    p.target = a.target;
    p.target_stride = a.target_stride;
    p.status = a.status;
    cudaError_t e = launch_kernel(kl_stats_kernel, dim3(p.chunks, p.G, (unsigned)bt), dim3(kTeam), 0, stream, p);
    if (e == cudaSuccess) e = launch_kernel(kl_totals_kernel, dim3((unsigned)bt), dim3(96), 0, stream, p);
    const int teams = p.G < kMaxTeams ? p.G : kMaxTeams;
    const size_t smem = kMaxTeams * sizeof(TeamSmem) + (size_t)p.G * kChunk * 4;
    if (e == cudaSuccess) {
        if (int rc = ensure_smem_limit((const void *)kl_target_kernel, smem, "cudaFuncSetAttribute(kl target)")) return rc;
        e = launch_kernel(kl_target_kernel, dim3(p.chunks, (unsigned)bt), dim3(teams * kTeam), smem, stream, p);
    }
    if (e == cudaSuccess) e = launch_kernel(kl_final_kernel, dim3((unsigned)bt), dim3(32), 0, stream, p);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "indexer KL launch");
}

}  // namespace dsa
