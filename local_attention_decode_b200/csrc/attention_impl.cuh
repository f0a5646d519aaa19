// attention_impl.cuh -- split-KV gather attention for decode, with a per-head
// sink (device code shared by the standalone attention kernels and the fused
// layer-step kernel).
//
// For each query head h of query (b, t), over a key set S (the selected
// top-k positions of a DSA layer, or the window {p-W+1..p} of an SWA layer):
//   s_i = sm_scale * Q[h] . K[row(b, i)][g],   g = h / (64 / G)
//   O[h] = sum_i e^{s_i} V[row(b, i)][g] / (sum_i e^{s_i} + e^{sink_h})
// ("Naive-N0.5-Flash: no full-attention layers, and a runtime built by AI":
// property table -- 64 query heads, qk dim 192, v dim 128, GQA4 / GQA8;
// "Inside a DSA layer" -- the main heads gather and attend to only the
// selected keys; the sink column in the softmax).
//
// attn_unit: a team of 4 warps takes 64 keys of one KV head, gathers their K
// and V rows (and the group's query rows) into shared memory with 16-byte
// asynchronous copies spread over the team's 128 threads (one bulk copy per
// row on the TMA engine issues more slowly: about 12 ns per copy on this GPU,
// 1.8 us for a unit's 144 rows), and computes for the
// 64/G query heads of that group  S = Q K^T  and  O = softmax_partial(S) V  on
// the tensor cores (mma.sync m16n8k16 bf16 -> fp32; the query heads of a group
// form the 16-row M dimension).  Each warp owns 16 keys; the four warps merge
// their (max, sum, O) in shared memory and the team writes one partial.
// combine_row_cta: log-sum-exp merge of the partials of all splits plus the
// sink term, normalisation, bf16 output and optional lse, one CTA per
// (query, head).
#pragma once

#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace attn {

constexpr int kChunk = kAttnChunk;   // keys per CTA
constexpr int kThreads = 128;
constexpr int kQS = DSA_QK_DIM + 8;  // padded smem row stride of Q and K (elements)
constexpr int kVS = DSA_V_DIM + 8;   // padded smem row stride of V
constexpr int kOS = DSA_V_DIM + 8;   // padded row stride (floats) of the O exchange: rows 8 banks apart
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
    const __nv_bfloat16 *Q;
    const __nv_bfloat16 *K;
    const __nv_bfloat16 *V;
    int G;
    const int32_t *block_table;
    int32_t max_pages, page_size;
    int64_t seq_stride, num_rows;
    const int32_t *idx;
    const int32_t *count;
    int idx_stride;
    const int32_t *q_pos;
    int window;
    int T;
    int n_teams;        // 64-key team chunks per CTA unit (1..4)
    int splits;         // CTA units per (query, KV head): ceil(max_keys / (64 * n_teams))
    float scale_log2;   // sm_scale * log2(e)
    float *part_o;
    float *part_ml;
    uint32_t *status;
    int padded;         // idx rows are full length, -1 past the selection: count is not read
};

struct Smem {
    __nv_bfloat16 q[16 * kQS];
    __nv_bfloat16 k[kChunk * kQS];
    __nv_bfloat16 v[kChunk * kVS];
    int64_t row[kChunk];
    float m[4][16];
    float l[4][16];
    float tm[16];   // the team's result: per head row, the max logit (log2 domain) ...
    float tl[16];   // ... and the sum of exp2(logit - max); its O is in the first 8 KB of k
};

static_assert(4 * 16 * kOS * 4 <= sizeof(Smem::k) + sizeof(Smem::v), "the O exchange fits in the K and V tiles");

// The teams' shared memory of a CTA: team t at base + t * stride.
struct TeamSmem {
    uint8_t *base;
    uint32_t stride;
    __device__ __forceinline__ Smem &operator[](int t) const { return *reinterpret_cast<Smem *>(base + t * stride); }
};

// Barrier of one 128-thread team.  The id is a run-time value, so that all
// teams of a CTA run one copy of the unit's code (one set of instruction-cache
// lines to fetch instead of one per team).
__device__ __forceinline__ void team_sync(int bar) {
    asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
// 8-byte copy (both addresses 8-byte aligned), cached in L1 on the way
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ bool key_row(const Params &p, int b, int64_t pos, int64_t *row) {
    if (pos < 0) return false;
    if (p.block_table == nullptr) {
        if (pos >= p.seq_stride) return false;
        *row = (int64_t)b * p.seq_stride + pos;
    } else {
        int64_t page = pos / p.page_size;
        if (page >= p.max_pages) return false;
        int32_t id = __ldg(p.block_table + (int64_t)b * p.max_pages + page);
        if (id < 0) return false;
        *row = (int64_t)id * p.page_size + pos % p.page_size;
    }
    return *row < p.num_rows;
}

// One team chunk: keys [chunk * 64, chunk * 64 + 64) of query bt and KV
// head g, by a team of 128 threads (tid 0..127) synchronised with the named
// barrier `bar`; leaves the chunk's result (per head row of the group: max
// logit, sum of exponentials, and the unnormalised O) in the team's shared
// memory (sm.tm, sm.tl, the first 16 x 128 floats of sm.k) for cta_merge.
// sel_smem: the query's selection (-1 padded, the p.padded layout) already
// in shared memory, read instead of p.idx.
// direct: a single-team unit (p.n_teams == 1) writes its result itself --
// the partial, or with one split the output -- with the arithmetic cta_merge
// would apply to it (a one-team merge multiplies by 2^0 = 1 and adds to 0:
// the same values), instead of leaving it in shared memory.
__device__ __forceinline__ void attn_unit(const Params &p, Smem &sm, int chunk, int g, int bt, int tid, int bar,
                                          const int32_t *sel_smem = nullptr, bool direct = false,
                                          const float *sink = nullptr, __nv_bfloat16 *O = nullptr,
                                          float *lse = nullptr) {
    const int b = bt / p.T;
    const int hpg = DSA_Q_HEADS / p.G;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- the key set of this split
    int n_total, win_lo = 0;
    if (p.idx) {
        n_total = p.padded ? p.idx_stride : min(__ldcg(p.count + bt), p.idx_stride);
    } else {
        const int32_t pq = __ldg(p.q_pos + bt);
        win_lo = max(0, pq - p.window + 1);
        n_total = pq >= 0 ? pq - win_lo + 1 : 0;
    }
    const int k0 = chunk * kChunk;
    const int nk = min(kChunk, n_total - k0);
    if (nk <= 0) {   // empty chunk: contributes nothing to the merge
        if (tid < 16) {
            sm.tm[tid] = -INFINITY;
            sm.tl[tid] = 0.f;
        }
        return;
    }

    // ---- positions -> cache rows (invalid ones are flagged and masked)
    if (tid < kChunk) {
        int64_t row = -1;
        if (tid < nk) {
            int64_t pos = sel_smem ? (int64_t)sel_smem[k0 + tid]
                          : p.idx  ? (int64_t)__ldcg(p.idx + (int64_t)bt * p.idx_stride + k0 + tid)
                                   : (int64_t)(win_lo + k0 + tid);
            if (p.padded && pos < 0) {
                row = -1;   // past the selection
            } else if (!key_row(p, b, pos, &row)) {
                flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
                row = -1;
            }
        }
        sm.row[tid] = row;
    }
    fence_proxy_async_smem();   // this thread's earlier use of the tiles, before the copies overwrite them
    team_sync(bar);
    // ---- the rows into shared memory by 16-byte asynchronous copies spread
    //      over the team's threads: K and Q in one group, V in the next
    const int G = p.G;
    constexpr int kKC = DSA_QK_DIM / 8, kVC = DSA_V_DIM / 8;   // 16-byte chunks per row
    for (int c = tid; c < kChunk * kKC; c += 128) {
        const int rr = c / kKC, cc = c % kKC;
        const int64_t row = sm.row[rr];
        __nv_bfloat16 *dst = sm.k + rr * kQS + cc * 8;
        if (row >= 0) cp_async16(dst, p.K + (row * G + g) * DSA_QK_DIM + cc * 8);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    for (int c = tid; c < 16 * kKC; c += 128) {
        const int rr = c / kKC, cc = c % kKC;
        __nv_bfloat16 *dst = sm.q + rr * kQS + cc * 8;
        if (rr < hpg) cp_async16(dst, p.Q + ((int64_t)bt * DSA_Q_HEADS + g * hpg + rr) * DSA_QK_DIM + cc * 8);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();
    for (int c = tid; c < kChunk * kVC; c += 128) {
        const int rr = c / kVC, cc = c % kVC;
        const int64_t row = sm.row[rr];
        __nv_bfloat16 *dst = sm.v + rr * kVS + cc * 8;
        if (row >= 0) cp_async16(dst, p.V + (row * G + g) * DSA_V_DIM + cc * 8);
        else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();
    cp_async_wait_group<1>();   // this thread's Q and K chunks
    team_sync(bar);             // and everyone's

    // ---- S = Q K^T for this warp's 16 keys (two n-tiles of 8)
    const int key0 = warp * 16;
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const uint32_t q_base = smem_u32(sm.q), k_base = smem_u32(sm.k), v_base = smem_u32(sm.v);
#pragma unroll
    for (int kk = 0; kk < DSA_QK_DIM / 16; ++kk) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(q_base + ((lane & 15) * kQS + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
        ldsm_x4(k_base + ((key0 + (lane >> 4) * 8 + (lane & 7)) * kQS + kk * 16 + ((lane >> 3) & 1) * 8) * 2,
                b0, b1, b2, b3);
        mma_bf16(s[0], a0, a1, a2, a3, b0, b1);
        mma_bf16(s[1], a0, a1, a2, a3, b2, b3);
    }

    // ---- partial softmax (log2 domain); rows g0 = lane/4 and g0 + 8
    const int g0 = lane >> 2, cq = lane & 3;
    float mrow[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = key0 + nt * 8 + cq * 2 + (e & 1);
            float v = (key < nk && sm.row[key] >= 0) ? s[nt][e] * p.scale_log2 : -INFINITY;
            s[nt][e] = v;
            mrow[e >> 1] = fmaxf(mrow[e >> 1], v);
        }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        mrow[r] = fmaxf(mrow[r], __shfl_xor_sync(0xffffffffu, mrow[r], 1));
        mrow[r] = fmaxf(mrow[r], __shfl_xor_sync(0xffffffffu, mrow[r], 2));
    }
    float lrow[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float m = mrow[e >> 1];
            const float pe = (m == -INFINITY) ? 0.f : exp2f(s[nt][e] - m);
            s[nt][e] = pe;
            lrow[e >> 1] += pe;
        }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
    }

    // ---- O_w = P V (P as the A operand straight from the S accumulators)
    const uint32_t pa0 = pack_bf16(s[0][0], s[0][1]), pa1 = pack_bf16(s[0][2], s[0][3]);
    const uint32_t pa2 = pack_bf16(s[1][0], s[1][1]), pa3 = pack_bf16(s[1][2], s[1][3]);
    float o[DSA_V_DIM / 8][4];
#pragma unroll
    for (int nt = 0; nt < DSA_V_DIM / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    cp_async_wait_group<0>();
    team_sync(bar);
#pragma unroll
    for (int dp = 0; dp < DSA_V_DIM / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(v_base + ((key0 + (lane & 7) + ((lane >> 3) & 1) * 8) * kVS + dp * 16 + (lane >> 4) * 8) * 2,
                  b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma_bf16(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
    }

    // ---- merge the four warps: (m, l) per row, then O through shared memory
    if (cq == 0) {
        sm.m[warp][g0] = mrow[0];
        sm.m[warp][g0 + 8] = mrow[1];
        sm.l[warp][g0] = lrow[0];
        sm.l[warp][g0 + 8] = lrow[1];
    }
    team_sync(bar);   // K/V tiles are no longer read: reuse them for the O exchange
    float *so = reinterpret_cast<float *>(sm.k);   // [4 warps][16 rows][kOS] (runs on into sm.v)
    float scale_row[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = g0 + 8 * r;
        float M = fmaxf(fmaxf(sm.m[0][row], sm.m[1][row]), fmaxf(sm.m[2][row], sm.m[3][row]));
        scale_row[r] = (mrow[r] == -INFINITY) ? 0.f : exp2f(mrow[r] - M);
    }
#pragma unroll
    for (int nt = 0; nt < DSA_V_DIM / 8; ++nt) {
        const int col = nt * 8 + cq * 2;
        float *d0 = so + (warp * 16 + g0) * kOS + col;
        float *d1 = so + (warp * 16 + g0 + 8) * kOS + col;
        *reinterpret_cast<float2 *>(d0) = make_float2(o[nt][0] * scale_row[0], o[nt][1] * scale_row[0]);
        *reinterpret_cast<float2 *>(d1) = make_float2(o[nt][2] * scale_row[1], o[nt][3] * scale_row[1]);
    }
    team_sync(bar);
    // each thread: one head row (tid / 8) and four 4-column pieces 32 apart
    // (eight threads read a row's 128 contiguous bytes at a time); the four
    // warps' scaled O summed in registers, then written over warp 0's slot
    const int row = tid >> 3, c0 = (tid & 7) * 4;
    float4 acc[4];
    float M = -INFINITY, L = 0.f;
    if (row < hpg) {
        M = fmaxf(fmaxf(sm.m[0][row], sm.m[1][row]), fmaxf(sm.m[2][row], sm.m[3][row]));
#pragma unroll
        for (int w = 0; w < 4; ++w)
            L += (sm.m[w][row] == -INFINITY) ? 0.f : sm.l[w][row] * exp2f(sm.m[w][row] - M);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 v = *reinterpret_cast<const float4 *>(so + (w * 16 + row) * kOS + c0 + 32 * c);
                acc[c].x += v.x; acc[c].y += v.y; acc[c].z += v.z; acc[c].w += v.w;
            }
        }
    }
    if (direct) {
        if (row < hpg) {
            const int64_t gw = (int64_t)bt * DSA_Q_HEADS + g * hpg + row;
            if (p.splits == 1) {
                const float sk = sink ? __ldg(sink + g * hpg + row) * kLog2e : -INFINITY;
                const float M2 = fmaxf(M, sk);
                float den = 0.f, w = 0.f;
                if (M2 != -INFINITY) {
                    w = (M == -INFINITY) ? 0.f : exp2f(M - M2);
                    den = L * w + (sink ? exp2f(sk - M2) : 0.f);
                }
                const float f = den > 0.f ? w / den : 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    __nv_bfloat16 *o = O + gw * DSA_V_DIM + c0 + 32 * c;
                    o[0] = __float2bfloat16_rn(acc[c].x * f);
                    o[1] = __float2bfloat16_rn(acc[c].y * f);
                    o[2] = __float2bfloat16_rn(acc[c].z * f);
                    o[3] = __float2bfloat16_rn(acc[c].w * f);
                }
                if (lse && (tid & 7) == 0) lse[gw] = den > 0.f ? (M2 + log2f(den)) / kLog2e : -INFINITY;
            } else {
                float *po = p.part_o + (gw * p.splits + chunk) * DSA_V_DIM;
#pragma unroll
                for (int c = 0; c < 4; ++c) *reinterpret_cast<float4 *>(po + c0 + 32 * c) = acc[c];
                if ((tid & 7) == 0) {
                    p.part_ml[(gw * p.splits + chunk) * 2 + 0] = M;
                    p.part_ml[(gw * p.splits + chunk) * 2 + 1] = L;
                }
            }
        }
        return;
    }
    team_sync(bar);
    if (row < hpg) {
#pragma unroll
        for (int c = 0; c < 4; ++c) *reinterpret_cast<float4 *>(so + row * kOS + c0 + 32 * c) = acc[c];
        if ((tid & 7) == 0) {
            sm.tm[row] = M;
            sm.tl[row] = L;
        }
    }
}

// The merge of the n_teams team chunks of one CTA unit (query bt, KV head g,
// unit `split`), by the threads t < n_teams * 128 of the CTA (after a barrier
// that follows the teams' attn_unit): thread t takes four columns of head
// rows t / 32, t / 32 + 4 n_teams, ... and merges the teams in order 0, 1, ...
// (teams with no key skipped).  With one unit per
// (query, KV head) (p.splits == 1) it finishes the output: the sink enters
// the denominator, O is normalised and written in bf16, with the lse.
// Otherwise it writes the unit's partial (O, max, sum) for the combine.
__device__ __forceinline__ void cta_merge(const Params &p, const TeamSmem &teams, int split, int g, int bt, int t,
                                          const float *sink, __nv_bfloat16 *O, float *lse) {
    const int hpg = DSA_Q_HEADS / p.G, c = (t & 31) * 4, row_step = p.n_teams * 4;
    for (int row = t >> 5; row < hpg; row += row_step) {
        float M = -INFINITY;
        for (int tm = 0; tm < p.n_teams; ++tm) M = fmaxf(M, teams[tm].tm[row]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float L = 0.f;
        for (int tm = 0; tm < p.n_teams; ++tm) {
            const float mt = teams[tm].tm[row];
            if (mt == -INFINITY) continue;
            const float w = exp2f(mt - M);
            const float4 v = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(teams[tm].k) +
                                                               row * kOS + c);
            acc.x += v.x * w; acc.y += v.y * w; acc.z += v.z * w; acc.w += v.w * w;
            L += teams[tm].tl[row] * w;
        }
        const int64_t gw = (int64_t)bt * DSA_Q_HEADS + g * hpg + row;
        if (p.splits == 1) {
            const float sk = sink ? __ldg(sink + g * hpg + row) * kLog2e : -INFINITY;
            const float M2 = fmaxf(M, sk);
            float den = 0.f, w = 0.f;
            if (M2 != -INFINITY) {
                w = (M == -INFINITY) ? 0.f : exp2f(M - M2);
                den = L * w + (sink ? exp2f(sk - M2) : 0.f);
            }
            const float f = den > 0.f ? w / den : 0.f;
            __nv_bfloat16 *o = O + gw * DSA_V_DIM + c;
            o[0] = __float2bfloat16_rn(acc.x * f);
            o[1] = __float2bfloat16_rn(acc.y * f);
            o[2] = __float2bfloat16_rn(acc.z * f);
            o[3] = __float2bfloat16_rn(acc.w * f);
            if (lse && c == 0) lse[gw] = den > 0.f ? (M2 + log2f(den)) / kLog2e : -INFINITY;
        } else {
            *reinterpret_cast<float4 *>(p.part_o + (gw * p.splits + split) * DSA_V_DIM + c) = acc;
            if (c == 0) {
                p.part_ml[(gw * p.splits + split) * 2 + 0] = M;
                p.part_ml[(gw * p.splits + split) * 2 + 1] = L;
            }
        }
    }
}

// One CTA unit: team tm < p.n_teams takes chunk split * n_teams + tm (team
// barriers bar0 + tm), then the n_teams * 128 threads merge after the
// barrier `cta_bar` (0 = __syncthreads, else a named barrier of those
// threads).  Exactly the threads t < n_teams * 128 call it.  The teams'
// shared memory may be reused after the call.
__device__ __forceinline__ void cta_unit(const Params &p, const TeamSmem &teams, int split, int g, int bt, int bar0,
                                         int cta_bar, const float *sink, __nv_bfloat16 *O, float *lse,
                                         const int32_t *sel_smem = nullptr) {
    const int t = threadIdx.x, tm = t >> 7;
    auto cta_sync = [&]() {
        if (cta_bar == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"r"(cta_bar), "r"(p.n_teams * 128) : "memory");
    };
    if (tm < p.n_teams) attn_unit(p, teams[tm], split * p.n_teams + tm, g, bt, t & 127, bar0 + tm, sel_smem);
    cta_sync();
    cta_merge(p, teams, split, g, bt, t, sink, O, lse);
    if (p.splits > 1) __threadfence();   // the partial is visible before any later signal of this CTA
    cta_sync();
}

// One unit taken by a single team (p.n_teams == 1): chunk `split` of query bt
// and KV head g, its partial (with one split: the output) written by the same
// 128 threads, which synchronise on the named barrier `bar` only, so that the
// teams of a CTA can work on different units at once.  On return the team's
// stores are done and, with several splits, released by thread 0 (tid 0): a
// flag that thread 0 then sets publishes the partial.
__device__ __forceinline__ void team_unit(const Params &p, Smem &sm, int split, int g, int bt, int tid, int bar,
                                          const float *sink, __nv_bfloat16 *O, float *lse,
                                          const int32_t *sel_smem = nullptr) {
    attn_unit(p, sm, split, g, bt, tid, bar, sel_smem, true, sink, O, lse);
    team_sync(bar);   // every thread's stores are done ...
    if (p.splits > 1 && tid == 0) __threadfence();   // ... and released, before thread 0 signals anything
}

// Merge of the splits of one (query, head) row gw by a whole CTA of NT
// threads (NT >= 8 * splits, splits <= 32): thread (split s, slice k) loads
// its split's 16-value slice and statistics, all loads issued at once; the
// weighted slices are summed over the splits through shared memory `red`
// (32 * 128 + 64 floats).
template <int NT>
__device__ void combine_row_cta(const float *part_o, const float *part_ml, int gw, int splits, const float *sink,
                                __nv_bfloat16 *O, float *lse, float *red) {
    static_assert(NT >= 256, "eight threads per split");
    const int t = threadIdx.x, s = t >> 3, k = t & 7;
    float *msm = red + 32 * DSA_V_DIM, *lsm = msm + 32;
    const float *ml = part_ml + (int64_t)gw * splits * 2;
    const float *po = part_o + ((int64_t)gw * splits + s) * DSA_V_DIM + k * 16;
    float m = -INFINITY, l = 0.f;
    float4 v[4];
    if (s < splits) {
        m = __ldcg(ml + 2 * s);
        l = __ldcg(ml + 2 * s + 1);
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldcg(reinterpret_cast<const float4 *>(po) + u);
    }
    if (k == 0 && s < 32) msm[s] = m;
    __syncthreads();
    const int h = gw % DSA_Q_HEADS;
    const float sk = sink ? __ldg(sink + h) * kLog2e : -INFINITY;
    float M = sk;
    for (int j = 0; j < splits; ++j) M = fmaxf(M, msm[j]);
    const float w = (M == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M);
    if (s < 32) {
        float *dst = red + s * DSA_V_DIM + k * 16;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 x = (s < splits && w != 0.f) ? v[u] : make_float4(0.f, 0.f, 0.f, 0.f);
            dst[4 * u + 0] = x.x * w;
            dst[4 * u + 1] = x.y * w;
            dst[4 * u + 2] = x.z * w;
            dst[4 * u + 3] = x.w * w;
        }
        if (k == 0) lsm[s] = (s < splits && w != 0.f) ? l * w : 0.f;
    }
    __syncthreads();
    if (t < DSA_V_DIM) {
        float acc = 0.f, L = (sink && M != -INFINITY) ? exp2f(sk - M) : 0.f;
        for (int j = 0; j < splits; ++j) {
            acc += red[j * DSA_V_DIM + t];
            L += lsm[j];
        }
        O[(int64_t)gw * DSA_V_DIM + t] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
        if (lse && t == 0) lse[gw] = (L > 0.f) ? (M + log2f(L)) / kLog2e : -INFINITY;
    }
    __syncthreads();
}

// Kernel parameters of the attention described by `a`.
inline Params make_params(const AttnArgs &a) {
    const dsa_kv_t *kv = a.kv;
    Params p;
    p.Q = a.Q;
    p.K = reinterpret_cast<const __nv_bfloat16 *>(kv->k);
    p.V = reinterpret_cast<const __nv_bfloat16 *>(kv->v);
    p.G = kv->num_kv_heads;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages;
    p.page_size = kv->page_size;
    p.seq_stride = kv->seq_stride;
    p.num_rows = kv->num_rows;
    p.idx = a.idx;
    p.count = a.count;
    p.idx_stride = a.idx_stride;
    p.q_pos = a.q_pos;
    p.window = a.window;
    p.T = a.T;
    p.n_teams = attn_teams(a.max_keys);
    p.splits = attn_splits(a.max_keys);
    p.scale_log2 = a.sm_scale * kLog2e;
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.status = a.status;
    p.padded = a.padded;
    return p;
}

}  // namespace attn
}  // namespace dsa
