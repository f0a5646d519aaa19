// indexer.cu -- the standalone lightning-indexer kernel (dsa_indexer_scores)
// and the host-side preparation shared with the fused layer-step (tensor maps,
// pipeline depth, grid).  The kernel body is in indexer_impl.cuh.
#include <algorithm>
#include <cstdio>
#include <cudaTypedefs.h>
#include <cstring>
#include <mutex>

#include "indexer_impl.cuh"
#include "kernels.h"

namespace dsa {
namespace indexer {

__global__ void __launch_bounds__(kThreads, 1)
indexer_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_ks,
               const __grid_constant__ CUtensorMap tmap_q, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    pdl_begin();
    // aligned by an offset from the array itself, so the compiler keeps the shared address space
    uint8_t *smem = smem_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) & 1023u)) & 1023u);
    run_indexer(&tmap_k, &tmap_ks, &tmap_q, p, smem, blockIdx.x, gridDim.x);
}

// --------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tensor-map encoding with a small cache: a decode loop calls the indexer with
// the same buffers step after step, and the encoding is host work on the
// critical path of every call.
struct MapKey {
    int device, dt, rank, swz;
    const void *base;
    uint64_t dims[2], strides[1];
    uint32_t box[2];
};

}  // namespace indexer

int make_tensor_map(const char *what, CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base,
                    const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz) {
    using namespace indexer;
    static std::mutex mu;
    static MapKey keys[32];
    static CUtensorMap maps[32];
    static int used = 0, next = 0;
    MapKey k;
    memset(&k, 0, sizeof k);
    cudaGetDevice(&k.device);
    k.dt = (int)dt;
    k.rank = rank;
    k.swz = (int)swz;
    k.base = base;
    for (int i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
    }
    if (rank > 1) k.strides[0] = strides_bytes[0];
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (memcmp(&keys[i], &k, sizeof k) == 0) {
                *map = maps[i];
                return DSA_OK;
            }
    }
    auto enc = get_encode();
    if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    uint32_t estr[2] = {1, 1};
    uint64_t no_strides[1] = {0};   // rank-1 maps take no strides; pass a valid pointer anyway
    CUresult r = enc(map, dt, rank, const_cast<void *>(base), dims, strides_bytes ? strides_bytes : no_strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(DSA_ERR_INVALID_ARG,
                    "tensor map encoding failed for %s (CUresult %d; base %p, dims %llu x %llu, box %u x %u)", what,
                    (int)r, base, (unsigned long long)dims[0], (unsigned long long)(rank > 1 ? dims[1] : 1),
                    box[0], rank > 1 ? box[1] : 1u);
    std::lock_guard<std::mutex> lock(mu);
    const int slot = used < 32 ? used++ : (next++ & 31);
    keys[slot] = k;
    maps[slot] = *map;
    return DSA_OK;
}

int prepare_indexer(const IndexerArgs &a, int hist_rows, int hist_row_words, uint32_t *hist_global,
                    size_t smem_budget, IndexerLaunch *out) {
    using namespace indexer;
    const dsa_kv_t *kv = a.kv;
    const DeviceInfo &dev = device_info();
    if (dev.num_sms <= 0) return fail(DSA_ERR_CUDA, "no CUDA device");

    const int T = a.T, N = 16 * T;
    const int R = kv->block_table ? std::min(kv->page_size, kTile) : kTile;
    {
        uint64_t dims[2] = {(uint64_t)kKeyBytes, (uint64_t)kv->num_rows};
        uint64_t strides[1] = {(uint64_t)kKeyBytes};
        uint32_t box[2] = {(uint32_t)kKeyBytes, (uint32_t)R};
        int rc = make_tensor_map("index keys", &out->tmap_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kv->index_k, dims, strides,
                          box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }
    {
        uint64_t dims[1] = {(uint64_t)kv->num_rows};
        uint32_t box[1] = {(uint32_t)R};
        int rc = make_tensor_map("index key scales", &out->tmap_ks, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, kv->index_k_scale,
                          dims, nullptr, box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc) return rc;
    }
    {
        uint64_t dims[2] = {(uint64_t)kKeyBytes, (uint64_t)a.B * T * 16};
        uint64_t strides[1] = {(uint64_t)kKeyBytes};
        uint32_t box[2] = {(uint32_t)kKeyBytes, (uint32_t)N};
        int rc = make_tensor_map("index queries", &out->tmap_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q8, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
    }

    // stages per pipeline: as many as fit next to the tables (2..8) in
    // smem_budget bytes (1 KB of which is alignment slack)
    const size_t budget = std::min<size_t>(smem_budget, dev.smem_optin) - 1024;
    const bool q_resident = a.B == 1;
    int S = kMaxStages;
    while (S > 2 && Layout(S, T, a.B, hist_rows, q_resident).total > budget) --S;
    Layout lay(S, T, a.B, hist_rows, q_resident);
    if (lay.total > budget)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "indexer shared memory does not fit (T=%d, B=%d)", T, a.B);
    out->smem = lay.total + 1024;

    Params &p = out->p;
    p.q_scale = a.q_scale;
    p.w = a.w;
    p.q_pos = a.q_pos;
    p.block_table = kv->block_table;
    p.max_pages = kv->max_pages;
    p.page_size = kv->page_size;
    p.seq_stride = kv->seq_stride;
    p.num_rows = kv->num_rows;
    p.B = a.B;
    p.T = T;
    p.Lmax = a.Lmax;
    p.scores = a.scores;
    p.scores_stride = a.scores_stride;
    p.status = a.status;
    p.stages = S;
    p.rows_per_load = R;
    p.groups = std::max(1, std::min(kMaxGroups, 512 / (kPipes * N)));
    p.acc_bufs = std::max(1, std::min(2, 512 / (kPipes * p.groups * N)));
    p.hist_rows = hist_rows;
    p.hist_row_words = hist_row_words;
    p.hist_global = hist_global;
    p.q_resident = q_resident ? 1 : 0;

    const int64_t max_tiles = (int64_t)a.B * ((a.Lmax + kTile - 1) / kTile);
    out->grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)dev.num_sms, max_tiles));
    return DSA_OK;
}

int launch_indexer(const IndexerArgs &a, cudaStream_t stream) {
    using namespace indexer;
    IndexerLaunch L;
    int rc = prepare_indexer(a, 0, 0, nullptr, device_info().smem_optin, &L);
    if (rc) return rc;
    if ((rc = ensure_smem_limit((const void *)indexer_kernel, L.smem, "cudaFuncSetAttribute(indexer)"))) return rc;
    // launched as a programmatic dependent: back-to-back calls overlap the launch with the previous tail
    cudaError_t e = launch_kernel_as(true, indexer_kernel, dim3(L.grid), dim3(kThreads), L.smem, stream, L.tmap_k,
                                     L.tmap_ks, L.tmap_q, L.p);
    if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
    return DSA_OK;
}

}  // namespace dsa
