// api.cu -- the C ABI of libdsa (declared in include/dsa.h): argument checks,
// workspace layout, and the launch sequences of each entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

static thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

const DeviceInfo &device_info() {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        static DeviceInfo none;
        return none;
    }
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo &d = cache[dev];
    if (d.device != dev) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
            d.num_sms = prop.multiProcessorCount;
            d.smem_optin = prop.sharedMemPerBlockOptin;
            d.device = dev;
        }
    }
    return d;
}

int ensure_smem_limit(const void *kernel, size_t bytes, const char *what) {
    struct Entry { const void *kernel; int device; size_t bytes; };
    static std::mutex mu;
    static Entry cache[64];
    static int used = 0;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    Entry *hit = nullptr;
    for (int i = 0; i < used; ++i)
        if (cache[i].kernel == kernel && cache[i].device == dev) hit = &cache[i];
    if (hit && hit->bytes >= bytes) return DSA_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    if (!hit && used < 64) hit = &cache[used++];
    if (hit) *hit = Entry{kernel, dev, bytes};
    return DSA_OK;
}

static thread_local bool g_pdl = false;
bool pdl_launches() { return g_pdl; }
void set_pdl_launches(bool on) { g_pdl = on; }

// Failure injection (dsa_debug_inject): process-wide, read at each launch.
static std::atomic<uint64_t *> g_trace_buf{nullptr};
static std::atomic<int64_t> g_trace_words{0};

uint64_t *phase_trace(int grid) {
    uint64_t *b = g_trace_buf.load();
    return b && g_trace_words.load() >= (int64_t)grid * DSA_TRACE_MARKS ? b : nullptr;
}

static std::atomic<int> g_inject_kind{DSA_INJECT_NONE};
static std::atomic<int64_t> g_inject_limit_ns{0};

BarrierCfg barrier_cfg() {
    BarrierCfg c;
    if (g_inject_kind.load() == DSA_INJECT_BARRIER_TIMEOUT) {
        c.limit_ns = (uint64_t)g_inject_limit_ns.load();
        c.extra = 1;
    }
    return c;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ----------------------------------------------------------- argument checks
static int check_common(int B, int T) {
    if (B < 1 || B > 1024) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B=%d outside [1, 1024]", B);
    if (T < 1 || T > DSA_MAX_T) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "T=%d outside [1, %d]", T, DSA_MAX_T);
    return DSA_OK;
}

static int check_kv_layout(const dsa_kv_t *kv) {
    if (!kv) return fail(DSA_ERR_INVALID_ARG, "kv is NULL");
    if (kv->num_rows < 1 || kv->num_rows >= (int64_t(1) << 31))
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "kv.num_rows=%lld outside [1, 2^31)", (long long)kv->num_rows);
    if (kv->block_table) {
        const int ps = kv->page_size;
        bool ok = ps >= 16 && ((ps <= 128 && 128 % ps == 0 && ps % 16 == 0) || (ps % 128 == 0));
        if (!ok) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "page_size=%d: need 16/32/64/128 or a multiple of 128", ps);
        if (kv->max_pages < 1) return fail(DSA_ERR_INVALID_ARG, "max_pages=%d < 1", kv->max_pages);
        if (kv->num_rows % ps) return fail(DSA_ERR_INVALID_ARG, "num_rows is not a multiple of page_size");
    } else {
        if (kv->seq_stride < 1) return fail(DSA_ERR_INVALID_ARG, "seq_stride=%lld < 1", (long long)kv->seq_stride);
    }
    return DSA_OK;
}

static int check_kv_backbone(const dsa_kv_t *kv) {
    int rc = check_kv_layout(kv);
    if (rc) return rc;
    if (!kv->k || !kv->v) return fail(DSA_ERR_INVALID_ARG, "kv.k / kv.v is NULL");
    if (!aligned16(kv->k) || !aligned16(kv->v)) return fail(DSA_ERR_INVALID_ARG, "kv.k / kv.v not 16-byte aligned");
    const int G = kv->num_kv_heads;
    if (G < 1 || DSA_Q_HEADS % G || DSA_Q_HEADS / G > 16)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "num_kv_heads=%d: need a divisor of 64 with at most 16 heads per group", G);
    return DSA_OK;
}

static int check_kv_index(const dsa_kv_t *kv) {
    int rc = check_kv_layout(kv);
    if (rc) return rc;
    if (!kv->index_k || !kv->index_k_scale) return fail(DSA_ERR_INVALID_ARG, "kv.index_k / index_k_scale is NULL");
    if (!aligned16(kv->index_k) || !aligned16(kv->index_k_scale))
        return fail(DSA_ERR_INVALID_ARG, "kv.index_k / index_k_scale not 16-byte aligned");
    return DSA_OK;
}

// The indexer's tensor copies start at row b * seq_stride of a contiguous
// cache; the fp32 scale copy needs that row to be a multiple of 4, so batched
// contiguous caches need seq_stride % 16 == 0 (paged caches start every copy
// at a page boundary).
static int check_index_stride(const dsa_kv_t *kv, int B) {
    if (!kv->block_table && B > 1 && kv->seq_stride % 16 != 0)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "contiguous index cache with B > 1 needs seq_stride %% 16 == 0 (got %lld)",
                    (long long)kv->seq_stride);
    return DSA_OK;
}

// ------------------------------------------------------------ workspace plan
struct WsPlan {
    size_t status = 0, scores = 0, idx = 0, count = 0, topk = 0, part_o = 0, part_ml = 0, cap_data = 0, total = 0;
    TopkPlan tp;
    FusedPlan fp;
    CapturePlan cp;
    size_t kl = 0;
};

static int plan_workspace(int op, int B, int T, int64_t Lmax, int top_k, WsPlan *w) {
    size_t off = kStatusBytes;
    w->status = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    switch (op) {
        case DSA_OP_INDEXER:
        case DSA_OP_PRODUCE:
            break;
        case DSA_OP_KL:
            w->kl = take(kl_workspace_bytes(B, T, Lmax));
            break;
        case DSA_OP_TOPK: {
            int rc = plan_topk(B, T, Lmax, top_k, &w->tp);
            if (rc) return rc;
            w->topk = take(w->tp.scratch_bytes);
            break;
        }
        case DSA_OP_SPARSE_ATTN:
        case DSA_OP_SWA_ATTN: {
            const int splits = attn_splits(top_k);
            const size_t rows = (size_t)B * T * DSA_Q_HEADS * splits;
            w->part_o = take(rows * DSA_V_DIM * 4);
            w->part_ml = take(rows * 2 * 4);
            break;
        }
        case DSA_OP_LAYER: {
            int rc = plan_topk(B, T, Lmax, top_k, &w->tp);
            if (rc) return rc;
            if ((rc = plan_fused(B, T, Lmax, top_k, &w->fp))) return rc;
            if ((rc = plan_capture(B, T, Lmax, top_k, &w->cp))) return rc;
            // the self-cleaning selection scratch first: its offset does not depend on the shape
            w->topk = take(std::max({w->tp.scratch_bytes, w->fp.ok ? w->fp.scratch_bytes : 0,
                                     w->cp.ok ? w->cp.scratch_bytes : 0}));
            w->cap_data = take(w->cp.ok ? w->cp.data_bytes : 0);
            w->scores = take((size_t)B * T * Lmax * 4);
            w->idx = take((size_t)B * T * top_k * 4);
            w->count = take((size_t)B * T * 4);
            const int splits = attn_splits(top_k);
            const size_t rows = (size_t)B * T * DSA_Q_HEADS * splits;
            w->part_o = take(rows * DSA_V_DIM * 4);
            w->part_ml = take(rows * 2 * 4);
            break;
        }
        default:
            return fail(DSA_ERR_INVALID_ARG, "unknown op %d", op);
    }
    w->total = off;
    return DSA_OK;
}

static int check_ws(void *ws, size_t ws_bytes, const WsPlan &w) {
    if (!ws) return fail(DSA_ERR_INVALID_ARG, "workspace is NULL");
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(DSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    if (ws_bytes < w.total)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, w.total);
    return DSA_OK;
}

template <class T>
static T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

static int record(void *const *events, int i, cudaStream_t s) {
    if (!events || !events[i]) return DSA_OK;
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "cudaEventRecord");
}

}  // namespace dsa

using namespace dsa;

extern "C" {

const char *dsa_last_error(void) { return g_err; }

int dsa_get_dims(int32_t *dims, int n) {
    if (!dims || n < 0 || n > 7) return fail(DSA_ERR_INVALID_ARG, "dims / n");
    const int32_t v[7] = {DSA_INDEX_HEADS, DSA_INDEX_DIM, DSA_Q_HEADS, DSA_QK_DIM, DSA_V_DIM, DSA_MAX_TOPK, DSA_MAX_T};
    for (int i = 0; i < n; ++i) dims[i] = v[i];
    return DSA_OK;
}

// Workspace of dsa_prefill: one layout for all of its query blocks
// (DSA_MAX_T tokens each, the last one possibly shorter), every region sized
// for the largest block, so that each block finds the self-cleaning selection
// scratch where the previous one left it clean.  full / tail: the plans the
// blocks run with (the tail's selection and launch plans, the shared offsets).
static int plan_prefill(int NQ, int64_t Lmax, int top_k, WsPlan *full, WsPlan *tail) {
    const int T0 = std::min(NQ, DSA_MAX_T), T1 = NQ % DSA_MAX_T ? NQ % DSA_MAX_T : T0;
    WsPlan a, b;
    int rc = plan_workspace(DSA_OP_LAYER, 1, T0, Lmax, top_k, &a);
    if (rc) return rc;
    if ((rc = plan_workspace(DSA_OP_LAYER, 1, T1, Lmax, top_k, &b))) return rc;
    // the layer layout puts the selection scratch right after the status word
    // in both plans; the later regions start after the larger of the two
    const size_t topk_end = std::max(a.scores, b.scores);
    const size_t shift = topk_end - a.scores;   // a is the larger block: move its later regions past both
    for (WsPlan *w : {&a}) {
        w->scores += shift;
        w->idx += shift;
        w->count += shift;
        w->part_o += shift;
        w->part_ml += shift;
        w->total += shift;
    }
    b.scores = a.scores;
    b.idx = a.idx;
    b.count = a.count;
    b.part_o = a.part_o;
    b.part_ml = a.part_ml;
    b.total = a.total;
    *full = a;
    *tail = b;
    return DSA_OK;
}

// The whole dsa_prefill workspace: the per-block layout (plan_prefill) at
// the start, then, when the tensor-core path applies, its region, then a
// one-token layer-step layout for the tokens it hands back (offsets shifted,
// the status word shared at offset 0).
struct PrefillLayout {
    WsPlan full, tail;        // the per-block path
    PrefillPlan cap;          // the tensor-core path (cap.ok)
    size_t cap_base = 0;
    WsPlan redo;              // one token at a time
    size_t total = 0;
};

static int plan_prefill_layout(int NQ, int64_t Lmax, int top_k, PrefillLayout *pl) {
    int rc = plan_prefill(NQ, Lmax, top_k, &pl->full, &pl->tail);
    if (rc) return rc;
    pl->total = pl->full.total;
    if ((rc = plan_prefill_capture(NQ, Lmax, top_k, &pl->cap))) return rc;
    if (!pl->cap.ok) return DSA_OK;
    pl->cap_base = align_up(pl->total, 256);
    size_t end = pl->cap_base + pl->cap.total;
    if ((rc = plan_workspace(DSA_OP_LAYER, 1, 1, Lmax, top_k, &pl->redo))) return rc;
    const size_t base = align_up(end, 256) - kStatusBytes;
    for (size_t *o : {&pl->redo.scores, &pl->redo.idx, &pl->redo.count, &pl->redo.topk, &pl->redo.part_o,
                      &pl->redo.part_ml, &pl->redo.cap_data, &pl->redo.total})
        *o += base;
    pl->total = pl->redo.total;
    return DSA_OK;
}

int dsa_workspace_size(int op, int B, int T, int64_t Lmax, int top_k, size_t *bytes) {
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    if (op == DSA_OP_PREFILL) {
        if (B != 1) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "DSA_OP_PREFILL takes one sequence (B = 1), got B=%d", B);
        if (T < 1) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "NQ=%d < 1", T);
        if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
        if (top_k < 1 || top_k > DSA_MAX_TOPK)
            return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
        PrefillLayout pl;
        int rc = plan_prefill_layout(T, Lmax, top_k, &pl);
        if (rc) return rc;
        *bytes = pl.total;
        return DSA_OK;
    }
    int rc = check_common(B, T);
    if (rc) return rc;
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (op != DSA_OP_INDEXER && (top_k < 1 || top_k > DSA_MAX_TOPK))
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k/window=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    WsPlan w;
    rc = plan_workspace(op, B, T, Lmax, top_k, &w);
    if (rc) return rc;
    *bytes = w.total;
    return DSA_OK;
}

int dsa_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws) return fail(DSA_ERR_INVALID_ARG, "workspace is NULL");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "cudaMemsetAsync(workspace)");
}

int dsa_check_device_status(void *ws, void *stream, int *status, uint32_t *flags) {
    if (!ws || !status) return fail(DSA_ERR_INVALID_ARG, "ws / status is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(&word, ws, 4, cudaMemcpyDeviceToHost);
    // the error bits are cleared by reading them; the re-initialisation bit
    // stays until dsa_workspace_init
    const uint32_t keep = word & kNeedsInitBit;
    if (e == cudaSuccess && word != keep) e = cudaMemcpy(ws, &keep, 4, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (flags) *flags = word;
    *status = (word & (1u << DSA_ERR_DEVICE_TIMEOUT))     ? DSA_ERR_DEVICE_TIMEOUT
              : (word & (1u << DSA_ERR_DEVICE_BAD_INDEX)) ? DSA_ERR_DEVICE_BAD_INDEX
                                                          : DSA_OK;
    return DSA_OK;
}

int dsa_layer_path_counts(void *ws, void *stream, uint32_t *fast, uint32_t *general) {
    if (!ws || !fast || !general) return fail(DSA_ERR_INVALID_ARG, "ws / fast / general is NULL");
    uint32_t w[2] = {0u, 0u};
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess)
        e = cudaMemcpy(w, static_cast<uint32_t *>(ws) + kPathCountWord, sizeof(w), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the path counters");
    *fast = w[0];
    *general = w[1];
    return DSA_OK;
}

int dsa_trace_phases(uint64_t *buf, int64_t words) {
    if (words < 0 || (!buf && words > 0)) return fail(DSA_ERR_INVALID_ARG, "trace buffer / words");
    g_trace_buf.store(nullptr);
    g_trace_words.store(buf ? words : 0);
    g_trace_buf.store(words > 0 ? buf : nullptr);
    return DSA_OK;
}

int dsa_debug_inject(int kind, int64_t wait_limit_ns) {
    if (kind == DSA_INJECT_NONE) {
        g_inject_kind.store(DSA_INJECT_NONE);
        g_inject_limit_ns.store(0);
        return DSA_OK;
    }
    if (kind != DSA_INJECT_BARRIER_TIMEOUT) return fail(DSA_ERR_INVALID_ARG, "unknown injection kind %d", kind);
    if (wait_limit_ns < 1000 || wait_limit_ns > 1000000000)
        return fail(DSA_ERR_INVALID_ARG, "wait_limit_ns=%lld outside [1e3, 1e9]", (long long)wait_limit_ns);
    g_inject_limit_ns.store(wait_limit_ns);
    g_inject_kind.store(kind);
    return DSA_OK;
}

int dsa_indexer_scores(const void *q8, const float *q_scale, const float *w, const dsa_kv_t *kv,
                       const int32_t *q_pos, int B, int T, int64_t Lmax, float *scores, int64_t scores_stride,
                       void *ws, size_t ws_bytes, void *stream) {
    if (!q8 || !q_scale || !w || !q_pos || !scores) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(q8)) return fail(DSA_ERR_INVALID_ARG, "q8 not 16-byte aligned");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (rc = check_kv_index(kv); rc) return rc;
    if (rc = check_index_stride(kv, B); rc) return rc;
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (scores_stride < Lmax) return fail(DSA_ERR_INVALID_ARG, "scores_stride < Lmax");
    WsPlan wp;
    if (rc = plan_workspace(DSA_OP_INDEXER, B, T, Lmax, 1, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    IndexerArgs a{static_cast<const uint8_t *>(q8), q_scale, w, kv, q_pos, B, T, Lmax, scores, scores_stride,
                  at<uint32_t>(ws, wp.status)};
    return launch_indexer(a, static_cast<cudaStream_t>(stream));
}

int dsa_index_produce(const void *k_in, const void *q_in, const float *ln_w, const float *ln_b, float ln_eps,
                      int rope_dim, double rope_base, const dsa_kv_t *kv, const int32_t *q_pos, int B, int T,
                      void *q8_out, float *q_scale_out, void *ws, size_t ws_bytes, void *stream) {
    if (!k_in || !ln_w || !ln_b || !q_pos) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (q_in && (!q8_out || !q_scale_out)) return fail(DSA_ERR_INVALID_ARG, "q_in given without q8_out / q_scale_out");
    if (!aligned16(k_in) || (q_in && (!aligned16(q_in) || !aligned16(q8_out))))
        return fail(DSA_ERR_INVALID_ARG, "k_in / q_in / q8_out not 16-byte aligned");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (rc = check_kv_index(kv); rc) return rc;
    if (rope_dim < 0 || rope_dim > DSA_INDEX_DIM || rope_dim % 2)
        return fail(DSA_ERR_INVALID_ARG, "rope_dim=%d: need an even number in [0, %d]", rope_dim, DSA_INDEX_DIM);
    if (!(rope_base > 1.0) || !std::isfinite(rope_base)) return fail(DSA_ERR_INVALID_ARG, "rope_base must be > 1");
    if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps)) return fail(DSA_ERR_INVALID_ARG, "ln_eps must be >= 0");
    WsPlan wp;
    if (rc = plan_workspace(DSA_OP_PRODUCE, B, T, 1, 1, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    ProduceArgs a{static_cast<const __nv_bfloat16 *>(k_in), static_cast<const __nv_bfloat16 *>(q_in), ln_w, ln_b,
                  ln_eps, rope_dim, rope_base, kv, q_pos, B, T, static_cast<uint8_t *>(q8_out), q_scale_out,
                  at<uint32_t>(ws, wp.status)};
    return launch_index_produce(a, static_cast<cudaStream_t>(stream));
}

int dsa_indexer_kl(const void *Q, const dsa_kv_t *kv, const float *scores, int64_t scores_stride,
                   const int32_t *q_pos, int B, int T, int64_t Lmax, float sm_scale, float *kl_out, float *target_out,
                   int64_t target_stride, void *ws, size_t ws_bytes, void *stream) {
    if (!Q || !scores || !q_pos || !kl_out) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(Q)) return fail(DSA_ERR_INVALID_ARG, "Q not 16-byte aligned");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (rc = check_kv_layout(kv); rc) return rc;
    if (!kv->k || !aligned16(kv->k)) return fail(DSA_ERR_INVALID_ARG, "kv.k is NULL or not 16-byte aligned");
    const int G = kv->num_kv_heads;
    if (G < 1 || DSA_Q_HEADS % G || DSA_Q_HEADS / G > 16)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "num_kv_heads=%d: need a divisor of 64 with at most 16 heads per group", G);
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (scores_stride < Lmax) return fail(DSA_ERR_INVALID_ARG, "scores_stride < Lmax");
    if (target_out && target_stride < Lmax) return fail(DSA_ERR_INVALID_ARG, "target_stride < Lmax");
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
    WsPlan wp;
    if (rc = plan_workspace(DSA_OP_KL, B, T, Lmax, 1, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    KlArgs a{static_cast<const __nv_bfloat16 *>(Q), kv, scores, scores_stride, q_pos, B, T, Lmax, sm_scale, kl_out,
             target_out, target_stride, at<void>(ws, wp.kl), at<uint32_t>(ws, wp.status)};
    return launch_indexer_kl(a, static_cast<cudaStream_t>(stream));
}

int dsa_topk_select(const float *scores, int64_t scores_stride, const int32_t *q_pos, int B, int T, int64_t Lmax,
                    int top_k, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes, void *stream) {
    if (!scores || !q_pos || !idx || !count) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (scores_stride < Lmax) return fail(DSA_ERR_INVALID_ARG, "scores_stride < Lmax");
    if (top_k < 1 || top_k > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    WsPlan wp;
    if (rc = plan_workspace(DSA_OP_TOPK, B, T, Lmax, top_k, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    return launch_topk(wp.tp, scores, scores_stride, q_pos, top_k, idx, count, at<uint32_t>(ws, wp.topk),
                       at<uint32_t>(ws, wp.status), static_cast<cudaStream_t>(stream));
}

static int attention_common(const void *Q, const dsa_kv_t *kv, const int32_t *idx, const int32_t *count,
                            const int32_t *q_pos, int window, int B, int T, int max_keys, const float *sink,
                            float sm_scale, void *O, float *lse, void *ws, size_t ws_bytes, void *stream, int op) {
    if (!Q || !O) return fail(DSA_ERR_INVALID_ARG, "Q / O is NULL");
    if (!aligned16(Q) || !aligned16(O)) return fail(DSA_ERR_INVALID_ARG, "Q / O not 16-byte aligned");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (rc = check_kv_backbone(kv); rc) return rc;
    if (max_keys < 1 || max_keys > DSA_MAX_TOPK)
        return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k/window=%d outside [1, %d]", max_keys, DSA_MAX_TOPK);
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
    WsPlan wp;
    if (rc = plan_workspace(op, B, T, 1, max_keys, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    AttnArgs a;
    a.Q = static_cast<const __nv_bfloat16 *>(Q);
    a.kv = kv;
    a.idx = idx;
    a.count = count;
    a.idx_stride = max_keys;
    a.q_pos = q_pos;
    a.window = window;
    a.B = B;
    a.T = T;
    a.max_keys = max_keys;
    a.sink = sink;
    a.sm_scale = sm_scale;
    a.O = static_cast<__nv_bfloat16 *>(O);
    a.lse = lse;
    a.part_o = at<float>(ws, wp.part_o);
    a.part_ml = at<float>(ws, wp.part_ml);
    a.status = at<uint32_t>(ws, wp.status);
    return launch_attention(a, static_cast<cudaStream_t>(stream));
}

int sparse_gqa_attn_decode(const void *Q, const dsa_kv_t *kv, const int32_t *idx, const int32_t *count, int B, int T,
                           int top_k, const float *sink, float sm_scale, void *O, float *lse, void *ws,
                           size_t ws_bytes, void *stream) {
    if (!idx || !count) return fail(DSA_ERR_INVALID_ARG, "idx / count is NULL");
    return attention_common(Q, kv, idx, count, nullptr, 0, B, T, top_k, sink, sm_scale, O, lse, ws, ws_bytes, stream,
                            DSA_OP_SPARSE_ATTN);
}

int swa_attn_decode(const void *Q, const dsa_kv_t *kv, const int32_t *q_pos, int B, int T, int window,
                    const float *sink, float sm_scale, void *O, float *lse, void *ws, size_t ws_bytes, void *stream) {
    if (!q_pos) return fail(DSA_ERR_INVALID_ARG, "q_pos is NULL");
    return attention_common(Q, kv, nullptr, nullptr, q_pos, window, B, T, window, sink, sm_scale, O, lse, ws, ws_bytes,
                            stream, DSA_OP_SWA_ATTN);
}

static int layer_run(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                     const int32_t *q_pos, int B, int T, int64_t Lmax, int top_k, const float *sink, float sm_scale,
                     void *O, float *lse, int32_t *idx_out, int32_t *count_out, void *ws, const WsPlan &wp,
                     cudaStream_t s, void *const *stage_events);

// Argument checks shared by dsa_layer_decode and dsa_prefill.
static int check_layer_args(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                            const int32_t *q_pos, int B, int T, int64_t Lmax, int top_k, float sm_scale, const void *O) {
    if (!q8 || !q_scale || !w || !Q || !q_pos || !O) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(q8) || !aligned16(Q) || !aligned16(O)) return fail(DSA_ERR_INVALID_ARG, "q8 / Q / O not 16-byte aligned");
    int rc = check_common(B, T);
    if (rc) return rc;
    if (rc = check_kv_index(kv); rc) return rc;
    if (rc = check_index_stride(kv, B); rc) return rc;
    if (rc = check_kv_backbone(kv); rc) return rc;
    if (Lmax < 1 || Lmax >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "Lmax outside [1, 2^31)");
    if (top_k < 1 || top_k > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
    return DSA_OK;
}

int dsa_layer_decode(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                     const int32_t *q_pos, int B, int T, int64_t Lmax, int top_k, const float *sink, float sm_scale,
                     void *O, float *lse, int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes,
                     void *stream, void *const *stage_events) {
    int rc = check_layer_args(q8, q_scale, w, Q, kv, q_pos, B, T, Lmax, top_k, sm_scale, O);
    if (rc) return rc;
    WsPlan wp;
    if (rc = plan_workspace(DSA_OP_LAYER, B, T, Lmax, top_k, &wp); rc) return rc;
    if (rc = check_ws(ws, ws_bytes, wp); rc) return rc;
    return layer_run(q8, q_scale, w, Q, kv, q_pos, B, T, Lmax, top_k, sink, sm_scale, O, lse, idx_out, count_out, ws,
                     wp, static_cast<cudaStream_t>(stream), stage_events);
}

// The layer-step on a checked workspace with plan wp.
static int layer_run(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                     const int32_t *q_pos, int B, int T, int64_t Lmax, int top_k, const float *sink, float sm_scale,
                     void *O, float *lse, int32_t *idx_out, int32_t *count_out, void *ws, const WsPlan &wp,
                     cudaStream_t s, void *const *stage_events) {
    int rc = DSA_OK;
    uint32_t *status = at<uint32_t>(ws, wp.status);
    float *scores = at<float>(ws, wp.scores);
    int32_t *idx = idx_out ? idx_out : at<int32_t>(ws, wp.idx);
    int32_t *count = count_out ? count_out : at<int32_t>(ws, wp.count);

    IndexerArgs ia{static_cast<const uint8_t *>(q8), q_scale, w, kv, q_pos, B, T, Lmax, scores, Lmax, status};
    if (wp.cp.ok || wp.fp.ok) {
        // one cooperative launch for the whole layer-step
        AttnArgs a;
        a.Q = static_cast<const __nv_bfloat16 *>(Q);
        a.kv = kv;
        a.idx = idx;
        a.count = count;
        a.idx_stride = top_k;
        a.q_pos = nullptr;
        a.window = 0;
        a.B = B;
        a.T = T;
        a.max_keys = top_k;
        a.sink = sink;
        a.sm_scale = sm_scale;
        a.O = static_cast<__nv_bfloat16 *>(O);
        a.lse = lse;
        a.part_o = at<float>(ws, wp.part_o);
        a.part_ml = at<float>(ws, wp.part_ml);
        a.status = status;
        a.padded = 1;   // the fused selection pads every idx row with -1
        if (wp.cp.ok)
            rc = launch_capture(wp.cp, ia, a, top_k, idx, count, at<uint8_t>(ws, wp.topk), at<uint8_t>(ws, wp.cap_data),
                                s, stage_events ? stage_events[0] : nullptr);
        if (!wp.cp.ok || rc == DSA_ERR_UNSUPPORTED_SHAPE)
            rc = wp.fp.ok ? launch_fused(wp.fp, ia, a, top_k, idx, count, at<uint32_t>(ws, wp.topk), s,
                                         stage_events ? stage_events[0] : nullptr)
                          : DSA_ERR_UNSUPPORTED_SHAPE;
        if (rc == DSA_OK) {
            for (int i = 1; i <= 4; ++i)
                if (rc = record(stage_events, i, s); rc) return rc;
            return DSA_OK;
        }
        if (rc != DSA_ERR_UNSUPPORTED_SHAPE) return rc;
        // the fused kernel does not fit this shape: run the separate kernels
    }
    if (rc = record(stage_events, 0, s); rc) return rc;
    if (rc = launch_indexer(ia, s); rc) return rc;
    if (rc = record(stage_events, 1, s); rc) return rc;
    if (rc = launch_topk(wp.tp, scores, Lmax, q_pos, top_k, idx, count, at<uint32_t>(ws, wp.topk), status, s); rc)
        return rc;
    if (rc = record(stage_events, 2, s); rc) return rc;
    AttnArgs a;
    a.Q = static_cast<const __nv_bfloat16 *>(Q);
    a.kv = kv;
    a.idx = idx;
    a.count = count;
    a.idx_stride = top_k;
    a.q_pos = nullptr;
    a.window = 0;
    a.B = B;
    a.T = T;
    a.max_keys = top_k;
    a.sink = sink;
    a.sm_scale = sm_scale;
    a.O = static_cast<__nv_bfloat16 *>(O);
    a.lse = lse;
    a.part_o = at<float>(ws, wp.part_o);
    a.part_ml = at<float>(ws, wp.part_ml);
    a.status = status;
    a.mid_event = stage_events ? stage_events[3] : nullptr;
    if (rc = launch_attention(a, s); rc) return rc;
    if (rc = record(stage_events, 4, s); rc) return rc;
    return DSA_OK;
}

}  // extern "C"

int dsa_prefill(const void *q8, const float *q_scale, const float *w, const void *Q, const dsa_kv_t *kv,
                const int32_t *q_pos, int NQ, int64_t Lmax, int top_k, const float *sink, float sm_scale, void *O,
                float *lse, int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes, void *stream) {
    if (NQ < 1) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "NQ=%d < 1", NQ);
    int rc = check_layer_args(q8, q_scale, w, Q, kv, q_pos, 1, std::min(NQ, DSA_MAX_T), Lmax, top_k, sm_scale, O);
    if (rc) return rc;
    PrefillLayout pl;
    if ((rc = plan_prefill_layout(NQ, Lmax, top_k, &pl))) return rc;
    if (ws_bytes < pl.total)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, pl.total);
    if ((rc = check_ws(ws, ws_bytes, pl.full))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t *q8b = static_cast<const uint8_t *>(q8);
    const __nv_bfloat16 *Qb = static_cast<const __nv_bfloat16 *>(Q);
    __nv_bfloat16 *Ob = static_cast<__nv_bfloat16 *>(O);
    auto tokens = [&](int t0, int T, const WsPlan &wp) {
        return layer_run(q8b + (size_t)t0 * DSA_INDEX_HEADS * DSA_INDEX_DIM, q_scale + (size_t)t0 * DSA_INDEX_HEADS,
                         w + (size_t)t0 * DSA_INDEX_HEADS, Qb + (size_t)t0 * DSA_Q_HEADS * DSA_QK_DIM, kv, q_pos + t0, 1,
                         T, Lmax, top_k, sink, sm_scale, Ob + (size_t)t0 * DSA_Q_HEADS * DSA_V_DIM,
                         lse ? lse + (size_t)t0 * DSA_Q_HEADS : nullptr, idx_out ? idx_out + (size_t)t0 * top_k : nullptr,
                         count_out ? count_out + t0 : nullptr, ws, wp, s, nullptr);
    };
    if (pl.cap.ok) {
        // the tensor-core path: the indexer as one contraction over all tokens
        PrefillArgs a{q8b, q_scale, w, Qb, kv, q_pos, Lmax, sink, sm_scale, Ob, lse, idx_out, count_out,
                      at<uint32_t>(ws, 0)};
        std::vector<int32_t> redo(NQ);
        int n_redo = 0;
        rc = run_prefill_capture(pl.cap, a, static_cast<uint8_t *>(ws) + pl.cap_base, s, redo.data(), &n_redo);
        if (rc == DSA_OK) {
            // the tokens whose candidates did not hold their selection: the decode layer-step, one by one
            for (int i = 0; i < n_redo; ++i)
                if ((rc = tokens(redo[i], 1, pl.redo))) return rc;
            return DSA_OK;
        }
        if (rc != DSA_ERR_UNSUPPORTED_SHAPE) return rc;
    }
    // one layer-step per block of DSA_MAX_T query tokens, on the one layout
    for (int t0 = 0; t0 < NQ; t0 += DSA_MAX_T) {
        const int T = std::min(DSA_MAX_T, NQ - t0);
        if ((rc = tokens(t0, T, T == DSA_MAX_T || T == NQ ? pl.full : pl.tail))) return rc;
    }
    return DSA_OK;
}

// ------------------------------------------------------------- the chain
// Checks of one chain step, exactly those its own entry point makes before
// enqueueing anything.
static int check_step(const dsa_layer_step_t &st) {
    WsPlan wp;
    int rc;
    if (st.kind == DSA_STEP_DSA) {
        if ((rc = check_layer_args(st.q8, st.q_scale, st.w, st.Q, st.kv, st.q_pos, st.B, st.T, st.Lmax, st.top_k,
                                   st.sm_scale, st.O)))
            return rc;
        if ((rc = plan_workspace(DSA_OP_LAYER, st.B, st.T, st.Lmax, st.top_k, &wp))) return rc;
        return check_ws(st.ws, st.ws_bytes, wp);
    }
    if (st.kind == DSA_STEP_SWA) {
        if (!st.q_pos) return fail(DSA_ERR_INVALID_ARG, "q_pos is NULL");
        if (!st.Q || !st.O) return fail(DSA_ERR_INVALID_ARG, "Q / O is NULL");
        if (!aligned16(st.Q) || !aligned16(st.O)) return fail(DSA_ERR_INVALID_ARG, "Q / O not 16-byte aligned");
        if ((rc = check_common(st.B, st.T))) return rc;
        if ((rc = check_kv_backbone(st.kv))) return rc;
        if (st.top_k < 1 || st.top_k > DSA_MAX_TOPK)
            return fail(DSA_ERR_UNSUPPORTED_SHAPE, "window=%d outside [1, %d]", st.top_k, DSA_MAX_TOPK);
        if (!(st.sm_scale > 0.f) || !std::isfinite(st.sm_scale))
            return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
        if ((rc = plan_workspace(DSA_OP_SWA_ATTN, st.B, st.T, 1, st.top_k, &wp))) return rc;
        return check_ws(st.ws, st.ws_bytes, wp);
    }
    return fail(DSA_ERR_INVALID_ARG, "unknown step kind %d", st.kind);
}

extern "C" int dsa_layer_chain(const dsa_layer_step_t *steps, int n_steps, void *stream) {
    if (!steps || n_steps < 1) return fail(DSA_ERR_INVALID_ARG, "steps is NULL or n_steps < 1");
    for (int i = 0; i < n_steps; ++i) {
        if (int rc = check_step(steps[i])) {
            char msg[512];
            snprintf(msg, sizeof msg, "%s", dsa_last_error());
            return fail(rc, "step %d: %s", i, msg);
        }
    }
    struct Pdl {   // the chained launch mode for this thread, restored on every exit
        Pdl() { set_pdl_launches(true); }
        ~Pdl() { set_pdl_launches(false); }
    } pdl;
    for (int i = 0; i < n_steps; ++i) {
        const dsa_layer_step_t &st = steps[i];
        int rc;
        if (st.kind == DSA_STEP_DSA)
            rc = dsa_layer_decode(st.q8, st.q_scale, st.w, st.Q, st.kv, st.q_pos, st.B, st.T, st.Lmax, st.top_k,
                                  st.sink, st.sm_scale, st.O, st.lse, st.idx_out, st.count_out, st.ws, st.ws_bytes,
                                  stream, nullptr);
        else
            rc = swa_attn_decode(st.Q, st.kv, st.q_pos, st.B, st.T, st.top_k, st.sink, st.sm_scale, st.O, st.lse,
                                 st.ws, st.ws_bytes, stream);
        if (rc) {
            char msg[512];
            snprintf(msg, sizeof msg, "%s", dsa_last_error());
            return fail(rc, "step %d: %s", i, msg);
        }
    }
    return DSA_OK;
}

// ------------------------------------------------- context-sharded decode
extern "C" int dsa_shard_positions(const int32_t *q_pos, int B, int T, int64_t shard_offset, int64_t shard_len,
                                   int32_t *q_pos_local, void *ws, size_t ws_bytes, void *stream) {
    if (!q_pos || !q_pos_local) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (int rc = check_common(B, T)) return rc;
    if (shard_offset < 0 || shard_len < 1) return fail(DSA_ERR_INVALID_ARG, "shard offset / length");
    WsPlan wp;
    if (int rc = plan_workspace(DSA_OP_PRODUCE, B, T, 1, 1, &wp)) return rc;
    if (int rc = check_ws(ws, ws_bytes, wp)) return rc;
    uint32_t *status = at<uint32_t>(ws, wp.status);
    // a query before the slice is flagged as a bad index in the status word
    return launch_shard_positions(q_pos, B * T, shard_offset, shard_len, q_pos_local, status,
                                  static_cast<cudaStream_t>(stream));
}

extern "C" int dsa_shard_candidates(const float *scores, int64_t scores_stride, const int32_t *idx, int B, int T,
                                    int top_k, int64_t shard_offset, float *cand_score, int32_t *cand_pos,
                                    void *stream) {
    if (!scores || !idx || !cand_score || !cand_pos) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (int rc = check_common(B, T)) return rc;
    if (top_k < 1 || top_k > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    if (shard_offset < 0) return fail(DSA_ERR_INVALID_ARG, "shard_offset < 0");
    return launch_shard_candidates(scores, scores_stride, idx, top_k, B * T, shard_offset, cand_score, cand_pos,
                                   static_cast<cudaStream_t>(stream));
}

extern "C" int dsa_shard_merge(const float *cand_score, const int32_t *cand_pos, int n_ranks, int B, int T, int top_k,
                               int64_t shard_offset, int64_t shard_len, int32_t *idx_out, int32_t *count_out,
                               int32_t *local_idx, int32_t *local_count, void *stream) {
    if (!cand_score || !cand_pos || !idx_out || !count_out) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if ((local_idx == nullptr) != (local_count == nullptr))
        return fail(DSA_ERR_INVALID_ARG, "local_idx and local_count go together");
    if (int rc = check_common(B, T)) return rc;
    if (n_ranks < 1 || n_ranks > 8) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "n_ranks=%d outside [1, 8]", n_ranks);
    if (top_k < 1 || top_k > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "top_k=%d outside [1, %d]", top_k, DSA_MAX_TOPK);
    return launch_shard_merge(cand_score, cand_pos, n_ranks, top_k, B * T, shard_offset, shard_len, idx_out, count_out,
                              local_idx, local_count, static_cast<cudaStream_t>(stream));
}

extern "C" int dsa_shard_combine(const void *O_all, const float *lse_all, int n_ranks, int B, int T, const float *sink,
                                 void *O, float *lse, void *stream) {
    if (!O_all || !lse_all || !O) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (int rc = check_common(B, T)) return rc;
    if (n_ranks < 1 || n_ranks > 8) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "n_ranks=%d outside [1, 8]", n_ranks);
    return launch_shard_combine(static_cast<const __nv_bfloat16 *>(O_all), lse_all, n_ranks, B * T, sink,
                                static_cast<__nv_bfloat16 *>(O), lse, static_cast<cudaStream_t>(stream));
}
