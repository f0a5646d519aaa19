// topk.cu -- the standalone top-k selection kernel (dsa_topk_select) and its
// launch plan.  The selection itself is in topk_impl.cuh.
#include <algorithm>

#include "kernels.h"
#include "topk_impl.cuh"

namespace dsa {
namespace topk {

constexpr int kThreads = 512;
constexpr int kMinChunk = 4096;             // keys per CTA below which a row is not split further
constexpr int kMaxCacheKeys = 32 * 1024;    // 128 KB of cached keys per CTA
constexpr int kVarMinRows = 16;             // above this many rows, CTAs per row follow the rows' lengths

__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    pdl_begin();
    const uint32_t status_at_entry = p.C > 1 ? load_status(p.status) : 0u;
    Shared<kThreads> *sh = reinterpret_cast<Shared<kThreads> *>(smem_raw);
    uint32_t *cache = reinterpret_cast<uint32_t *>(smem_raw + sizeof(Shared<kThreads>));
    if (p.var_c) {
        int row, c, C;
        row_of_cta<kThreads>(p, sh, &row, &c, &C);
        if (row >= 0) select_row<kThreads>(p, sh, cache, row, c, C, false, status_at_entry);
        return;
    }
    select_row<kThreads>(p, sh, cache, blockIdx.x / p.C, blockIdx.x % p.C, p.C, false, status_at_entry);
}

}  // namespace topk

int plan_topk(int B, int T, int64_t Lmax, int top_k, TopkPlan *plan, size_t max_scratch_bytes) {
    using namespace topk;
    const DeviceInfo &dev = device_info();
    plan->rows = B * T;
    plan->threads = kThreads;
    plan->Lmax = Lmax;
    int C = 1;
    plan->var_c = false;
    if (dev.num_sms > 0 && Lmax > top_k) {
        // rows * C CTAs, at most one per SM: the cooperative launch below
        // guarantees they are all resident together (their row barriers wait
        // on one another)
        int co_resident = dev.num_sms;
        C = (int)std::max<int64_t>(1, std::min<int64_t>(co_resident / std::max(1, plan->rows),
                                                       (Lmax + kMinChunk - 1) / kMinChunk));
        // many rows of unequal length: CTAs in proportion to each row's length
        // (decided on the device from the positions), up to grid - rows + 1 per row
        if (plan->rows > kVarMinRows && plan->rows < co_resident && Lmax > 2 * kMinChunk) {
            plan->var_c = true;
            C = co_resident - plan->rows + 1;
        }
    }
    int64_t chunk = ((Lmax + C - 1) / C + 3) & ~int64_t(3);
    if (plan->var_c) chunk = kMaxCacheKeys;   // slices depend on the lengths: the most the cache holds
    plan->ctas_per_row = C;
    plan->cache_keys = (int)std::min<int64_t>(chunk, kMaxCacheKeys);
    plan->list_cap = 0;
    plan->smem_list = 0;
    plan->cand_cap = 0;
    plan->scratch_bytes = 0;
    if (C > 1) {
        int cap = kListCap;
        const size_t fixed = (size_t)plan->rows * scratch_words(C, 0) * 4;
        if (fixed > max_scratch_bytes) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top-k scratch exceeds %zu bytes", max_scratch_bytes);
        cap = (int)std::min<size_t>(cap, (max_scratch_bytes - fixed) / ((size_t)plan->rows * 8));
        plan->list_cap = cap & ~3;
        // room for the kernel's static shared memory (under 1 KB) stays free
        const size_t used = sizeof(Shared<kThreads>) + (size_t)plan->cache_keys * 4 + 1024;
        size_t room = dev.smem_optin > used ? (dev.smem_optin - used) / 8 : 0;   // (key, position) pairs
        plan->smem_list = (int)std::min<size_t>({(size_t)plan->list_cap, (size_t)kSmemList, room});
        room -= plan->smem_list;
        plan->cand_cap = (int)(std::min<size_t>(kCandCap, room) / (kThreads / 32) * (kThreads / 32));
        plan->scratch_bytes = (size_t)plan->rows * scratch_words(C, plan->list_cap) * 4;
    }
    plan->smem = sizeof(Shared<kThreads>) +
                 ((size_t)plan->cache_keys + 2 * (size_t)plan->smem_list + 2 * (size_t)plan->cand_cap) * 4;
    return DSA_OK;
}

int launch_topk(const TopkPlan &plan, const float *scores, int64_t stride, const int32_t *q_pos, int top_k,
                int32_t *idx, int32_t *count, uint32_t *scratch, uint32_t *status, cudaStream_t stream, float *kth) {
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
    p.scratch_row_words = scratch_words(plan.ctas_per_row, plan.list_cap);
    p.status = status;
    p.cache_keys = plan.cache_keys;
    p.list_cap = plan.list_cap;
    p.smem_list = plan.smem_list;
    p.cand_cap = plan.cand_cap;
    p.Lmax = plan.Lmax;
    p.bar = barrier_cfg();
    p.kth = kth;
    p.var_c = plan.var_c ? 1 : 0;
    if (int rc = ensure_smem_limit((const void *)topk_kernel, plan.smem, "cudaFuncSetAttribute(topk)")) return rc;
    cudaError_t e;
    const unsigned grid = plan.var_c ? (unsigned)device_info().num_sms : (unsigned)(plan.rows * plan.ctas_per_row);
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
        e = launch_kernel(topk_kernel, dim3(grid), dim3(kThreads), plan.smem, stream, p);
    }
    if (e != cudaSuccess) return cuda_fail(e, "topk launch");
    return DSA_OK;
}

}  // namespace dsa
