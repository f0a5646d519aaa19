// noalloc.cu -- top-k selection for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: code that runs inside a
// host framework which owns all device memory and forbids further
// allocation once it is initialised, real-time loops that must not touch the
// allocator after start-up, or plug-ins that receive only input and output
// pointers.  dsa_topk_select_noalloc serves them with the same selection
// kernel as dsa_topk_select, taking its scratch from a fixed array in device
// memory that the library itself declares.  The array lives on every GPU that
// loads the library until the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;   // 2 MiB per device

// Device-side scratch shared by every call on a device.  In host code this
// name is only a handle for the runtime; its device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
static int static_scratch_address(void **out) {
    static std::mutex mu;
    static void *cached[64] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "device index %d not supported", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        cached[dev] = p;
    }
    *out = cached[dev];
    return DSA_OK;
}

}  // namespace dsa

using namespace dsa;

extern "C" int dsa_topk_select_noalloc(const float *scores, int64_t scores_stride, const int32_t *q_pos, int B, int T,
                                       int64_t Lmax, int top_k, int32_t *idx, int32_t *count, void *stream) {
    if (!scores || !q_pos || !idx || !count) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (B < 1 || B > 1024) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B=%d outside [1, 1024]", B);
    if (T < 1 || T > DSA_MAX_T) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "T=%d outside [1, %d]", T, DSA_MAX_T);
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (scores_stride < Lmax) return fail(DSA_ERR_INVALID_ARG, "scores_stride < Lmax");
    if (top_k < 1 || top_k > DSA_MAX_TOPK)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    TopkPlan plan;
    int rc = plan_topk(B, T, Lmax, top_k, &plan, kStaticScratchBytes - kStatusBytes);
    if (rc) return rc;
    const size_t need = kStatusBytes + plan.scratch_bytes;
    if (need > kStaticScratchBytes)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE,
                    "dsa_topk_select_noalloc: this call needs %zu bytes of scratch; the static scratch holds %zu "
                    "(use dsa_topk_select with a workspace)",
                    need, kStaticScratchBytes);
    void *base = nullptr;
    if ((rc = static_scratch_address(&base))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: clear the status word and
    // the cross-CTA histograms, counts and barrier words before this call.
    cudaError_t e = cudaMemsetAsync(base, 0, need, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(static scratch)");
    uint8_t *b8 = static_cast<uint8_t *>(base);
    return launch_topk(plan, scores, scores_stride, q_pos, top_k, idx, count,
                       reinterpret_cast<uint32_t *>(b8 + kStatusBytes), reinterpret_cast<uint32_t *>(b8), s);
}
