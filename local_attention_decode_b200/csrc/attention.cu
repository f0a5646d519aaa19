// attention.cu -- standalone split-KV attention kernels (sparse_gqa_attn_decode,
// swa_attn_decode) and their launcher.  The device code is in
// attention_impl.cuh.
#include <algorithm>

#include "attention_impl.cuh"

namespace dsa {
namespace attn {

constexpr size_t kTeamSmem = (sizeof(Smem) + 127) & ~size_t(127);

// One CTA unit per block: n_teams teams of 128 threads (the block), grid
// (units per query and KV head, KV heads, queries).
__global__ void __launch_bounds__(kAttnMaxTeams * kThreads)
gather_attn_kernel(const Params p, const float *sink, __nv_bfloat16 *O, float *lse) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    pdl_begin();
    const TeamSmem teams{smem_raw, (uint32_t)kTeamSmem};
    cta_unit(p, teams, blockIdx.x, blockIdx.y, blockIdx.z, 1, 0, sink, O, lse);
}

// One CTA per (query, head), as in the fused layer-step (same arithmetic).
constexpr int kCombineThreads = 256;
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float *part_o, const float *part_ml, int splits, const float *sink, __nv_bfloat16 *O,
               float *lse) {
    __shared__ float red[32 * DSA_V_DIM + 64];
    pdl_begin();
    combine_row_cta<kCombineThreads>(part_o, part_ml, blockIdx.x, splits, sink, O, lse, red);
}

}  // namespace attn

size_t attn_partial_bytes(int B, int T, int max_keys) {
    const int splits = attn_splits(max_keys);
    const size_t rows = (size_t)B * T * DSA_Q_HEADS * splits;
    return rows * DSA_V_DIM * 4 + rows * 2 * 4 + 512;
}

int launch_attention(const AttnArgs &a, cudaStream_t stream) {
    using namespace attn;
    Params p = make_params(a);
    const size_t smem = p.n_teams * kTeamSmem;
    if (int rc = ensure_smem_limit((const void *)gather_attn_kernel, smem, "cudaFuncSetAttribute(attention)")) return rc;
    cudaError_t e;
    dim3 grid(p.splits, p.G, a.B * a.T);
    e = launch_kernel(gather_attn_kernel, grid, dim3(p.n_teams * kThreads), smem, stream, p, a.sink, a.O, a.lse);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    if (a.mid_event) {
        e = cudaEventRecord(static_cast<cudaEvent_t>(a.mid_event), stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    if (p.splits == 1) return DSA_OK;   // the CTA units wrote the output
    const int rows = a.B * a.T * DSA_Q_HEADS;
    e = launch_kernel(combine_kernel, dim3(rows), dim3(kCombineThreads), 0, stream, (const float *)a.part_o,
                      (const float *)a.part_ml, p.splits, a.sink, a.O, a.lse);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return DSA_OK;
}

}  // namespace dsa
