// produce.cu -- the indexer's inputs for new tokens: the index key of each
// token normalised (LayerNorm), turned by partial RoPE, quantised to e4m3
// with a per-token scale and written into the index-key cache at the token's
// position; the index queries turned by the same partial RoPE and quantised
// with one scale per token.  ("Naive-N0.5-Flash: no full-attention layers,
// and a runtime built by AI", section "Inside a DSA layer: the lightning
// indexer": the key is normalised, given RoPE, and both sides are rounded to
// fp8_e4m3; the inherited attention block's partial RoPE, and its rope base
// of 10,000,000 on the sparse layers, are in the same section.)
//
// One CTA per token, 17 warps: warp h < 16 holds index-query head h, warp 16
// the index key; each lane holds 4 of the 128 dims.  Rotary pairs are
// (i, i + rot/2) for i < rot/2 (the rotate-half arrangement), angle
// pos * base^(-2i/rot) computed in double (at positions near 2^20 an fp32
// angle would be off by hundredths of a radian), the rotation in fp32.  The
// scale is amax / 448 in fp32, value / scale in fp32, and the e4m3 code is
// the hardware's round-to-nearest-even conversion with saturation at 448.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace produce {

constexpr int kWarps = DSA_INDEX_HEADS + 1;
constexpr int kThreads = 32 * kWarps;
constexpr int kD = DSA_INDEX_DIM;

struct Params {
    const __nv_bfloat16 *k_in;   // [rows][128]
    const __nv_bfloat16 *q_in;   // [rows][16][128] or null
    const float *ln_w, *ln_b;    // [128]
    float ln_eps;
    int rot;
    double log_base;
    const int32_t *q_pos;        // [rows]
    int T;
    // the index-key cache
    uint8_t *index_k;
    float *index_k_scale;
    const int32_t *block_table;
    int32_t max_pages, page_size;
    int64_t seq_stride, num_rows;
    // index-query outputs
    uint8_t *q8;                 // [rows][16][128]
    float *q_scale;              // [rows][16]
    uint32_t *status;
};

// Partial RoPE of this lane's 4 dims (d0 .. d0 + 3) of a 128-vector whose
// values are all in `row` (shared), in place into v.
__device__ __forceinline__ void rope4(float (&v)[4], const float *row, int d0, int rot, double log_base, int64_t pos) {
    const int h = rot / 2;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int d = d0 + u;
        if (d < rot) {
            const int i = d < h ? d : d - h;
            const double ang = (double)pos * exp(-2.0 * (double)i / (double)rot * log_base);
            double s, c;
            sincos(ang, &s, &c);
            const float cf = (float)c, sf = (float)s;
            if (d < h) v[u] = row[d] * cf - row[d + h] * sf;   // x_i cos - x_{i+h} sin
            else v[u] = row[d] * cf + row[d - h] * sf;         // x_{i+h} cos + x_i sin
        }
    }
}

__device__ __forceinline__ uint32_t pack_e4m3(const float (&v)[4], float scale) {
    uint32_t out = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(v[u] / scale, __NV_SATFINITE, __NV_E4M3);
        out |= (uint32_t)c << (8 * u);
    }
    return out;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__global__ void __launch_bounds__(kThreads)
index_produce_kernel(const Params p) {
    __shared__ float rows_s[kWarps][kD];
    __shared__ float amax_s[kWarps];
    pdl_begin();
    const int tok = blockIdx.x, warp = warp_id(), lane = lane_id(), d0 = 4 * lane;
    const int64_t pos = __ldg(p.q_pos + tok);
    float v[4];
    if (warp < DSA_INDEX_HEADS) {
        // ---- index-query head `warp`
        if (p.q_in) {
            const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.q_in + ((int64_t)tok * DSA_INDEX_HEADS + warp) * kD + d0));
            const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
            const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
            v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
        } else {
            v[0] = v[1] = v[2] = v[3] = 0.f;
        }
    } else {
        // ---- the index key: LayerNorm over the 128 dims
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.k_in + (int64_t)tok * kD + d0));
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
        const float mean = warp_sum((v[0] + v[1]) + (v[2] + v[3])) / (float)kD;
        float sq = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) sq += (v[u] - mean) * (v[u] - mean);
        const float var = warp_sum(sq) / (float)kD;
        const float inv = 1.0f / sqrtf(var + p.ln_eps);
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = (v[u] - mean) * inv * __ldg(p.ln_w + d0 + u) + __ldg(p.ln_b + d0 + u);
    }
    // ---- partial RoPE (partners may sit in other lanes: through shared memory)
#pragma unroll
    for (int u = 0; u < 4; ++u) rows_s[warp][d0 + u] = v[u];
    __syncwarp();
    rope4(v, rows_s[warp], d0, p.rot, p.log_base, pos);
    const float am = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
    if (lane == 0) amax_s[warp] = am;
    __syncthreads();
    if (warp == DSA_INDEX_HEADS) {
        // ---- key: one scale, codes into the cache row of (sequence, pos)
        const float scale = am > 0.f ? am / 448.0f : 1.0f;
        const int b = tok / p.T;
        bool ok = pos >= 0;
        int64_t row = 0;
        if (ok) {
            if (p.block_table == nullptr) {
                ok = pos < p.seq_stride;
                row = (int64_t)b * p.seq_stride + pos;
            } else {
                const int64_t page = pos / p.page_size;
                ok = page < p.max_pages;
                const int32_t id = ok ? __ldg(p.block_table + (int64_t)b * p.max_pages + page) : -1;
                ok = ok && id >= 0;
                row = (int64_t)id * p.page_size + pos % p.page_size;
            }
            ok = ok && row < p.num_rows;
        }
        if (!ok) {
            if (lane == 0) flag_error(p.status, DSA_ERR_DEVICE_BAD_INDEX);
        } else {
            reinterpret_cast<uint32_t *>(p.index_k + row * kD)[lane] = pack_e4m3(v, scale);
            if (lane == 0) p.index_k_scale[row] = scale;
        }
    } else if (p.q_in) {
        // ---- query: one scale for the token's 16 heads
        float qa = amax_s[0];
#pragma unroll
        for (int h = 1; h < DSA_INDEX_HEADS; ++h) qa = fmaxf(qa, amax_s[h]);
        const float scale = qa > 0.f ? qa / 448.0f : 1.0f;
        reinterpret_cast<uint32_t *>(p.q8 + ((int64_t)tok * DSA_INDEX_HEADS + warp) * kD)[lane] = pack_e4m3(v, scale);
        if (lane == 0) p.q_scale[(int64_t)tok * DSA_INDEX_HEADS + warp] = scale;
    }
}

}  // namespace produce

int launch_index_produce(const ProduceArgs &a, cudaStream_t stream) {
    using namespace produce;
    Params p;
    p.k_in = a.k_in;
    p.q_in = a.q_in;
    p.ln_w = a.ln_w;
    p.ln_b = a.ln_b;
    p.ln_eps = a.ln_eps;
    p.rot = a.rope_dim;
    p.log_base = log(a.rope_base);
    p.q_pos = a.q_pos;
    p.T = a.T;
    p.index_k = static_cast<uint8_t *>(const_cast<void *>(a.kv->index_k));
    p.index_k_scale = const_cast<float *>(a.kv->index_k_scale);
    p.block_table = a.kv->block_table;
    p.max_pages = a.kv->max_pages;
    p.page_size = a.kv->page_size;
    p.seq_stride = a.kv->seq_stride;
    p.num_rows = a.kv->num_rows;
    p.q8 = a.q8;
    p.q_scale = a.q_scale;
    p.status = a.status;
    cudaError_t e = launch_kernel(index_produce_kernel, dim3(a.B * a.T), dim3(kThreads), 0, stream, p);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "index producer launch");
}

}  // namespace dsa
