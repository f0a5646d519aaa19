// attention.cu -- standalone split-KV attention kernels (sparse_gqa_attn_decode,
// swa_attn_decode) and their launcher.  The device code is in
// attention_impl.cuh.
#include <algorithm>

#include "attention_impl.cuh"

namespace dsa {
namespace attn {

__global__ void __launch_bounds__(kThreads)
gather_attn_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    attn_unit(p, sm, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x, 0);
}

// One CTA per (query, head), as in the fused layer-step (same arithmetic).
constexpr int kCombineThreads = 256;
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float *part_o, const float *part_ml, int splits, const float *sink, __nv_bfloat16 *O,
               float *lse) {
    __shared__ float red[32 * DSA_V_DIM + 64];
    combine_row_cta<kCombineThreads>(part_o, part_ml, blockIdx.x, splits, sink, O, lse, red);
}

}  // namespace attn

size_t attn_partial_bytes(int B, int T, int max_keys) {
    const int splits = (max_keys + kAttnChunk - 1) / kAttnChunk;
    const size_t rows = (size_t)B * T * DSA_Q_HEADS * splits;
    return rows * DSA_V_DIM * 4 + rows * 2 * 4 + 512;
}

int launch_attention(const AttnArgs &a, cudaStream_t stream) {
    using namespace attn;
    Params p = make_params(a);
    const size_t smem = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(gather_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attention)");
    dim3 grid(p.splits, p.G, a.B * a.T);
    gather_attn_kernel<<<grid, kThreads, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    if (a.mid_event) {
        e = cudaEventRecord(static_cast<cudaEvent_t>(a.mid_event), stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    const int rows = a.B * a.T * DSA_Q_HEADS;
    combine_kernel<<<rows, kCombineThreads, 0, stream>>>(a.part_o, a.part_ml, p.splits, a.sink, a.O, a.lse);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return DSA_OK;
}

}  // namespace dsa
