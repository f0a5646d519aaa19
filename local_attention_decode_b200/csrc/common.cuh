// common.cuh -- sm_100a building blocks shared by the libdsa kernels:
// mbarriers with bounded waits, TMA tensor loads, tcgen05 (TMEM alloc, MMA,
// commit, loads), the device status word, and the host-side status codes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace hold a 32-bit status word: bit
// (1 << code) is set for each kind of device-side error seen.
constexpr size_t kStatusBytes = 256;
// Words 1 and 2 of the workspace header: layer-steps the one-barrier kernel
// ran on its fast path and on its general path (see dsa_layer_path_counts).
constexpr int kPathCountWord = 1;

__device__ __forceinline__ void flag_error(uint32_t *status, int code) {
    if (status) atomicOr(status, 1u << code);
}

// Bit 31 of the status word: a cross-CTA wait ran out, so the workspace's
// self-cleaning scratch (barrier counters, histograms, lists) may hold a
// partial state.  Kernels that use that scratch refuse to run on it (they set
// the timeout bit again and return) until dsa_workspace_init zeroes it.
constexpr uint32_t kNeedsInitBit = 1u << 31;

__device__ __forceinline__ void flag_timeout(uint32_t *status) {
    if (status) atomicOr(status, (1u << DSA_ERR_DEVICE_TIMEOUT) | kNeedsInitBit);
}

// Status word as seen at kernel entry (read through L2; a plain load issued
// early, so that its latency overlaps the kernel's first phase).
__device__ __forceinline__ uint32_t load_status(const uint32_t *status) {
    return status ? __ldcg(status) : 0u;
}

// Time limit of every spin-wait in device code (nanoseconds of the global
// timer): far beyond any legitimate wait in these kernels, short enough that a
// broken wait ends the kernel with an error status instead of a hang.
constexpr uint64_t kWaitLimitNs = 2000000000ull;


__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Cross-CTA barrier settings of one launch: the time limit of its waits and a
// number of arrivals added to every barrier's target.  `extra` is 0 except
// under the library's failure injection (dsa_debug_inject), where it makes
// the first barrier wait for an arrival that never comes, so that the wait
// runs out after `limit_ns` and the kernel takes its error path.
struct BarrierCfg {
    uint64_t limit_ns = kWaitLimitNs;
    uint32_t extra = 0;
};
// The settings for a launch made now (host side; see dsa_debug_inject).
BarrierCfg barrier_cfg();
// The phase-trace buffer set by dsa_trace_phases when it holds `grid` CTAs'
// marks, else NULL (host).
uint64_t *phase_trace(int grid);

// Reduction with release semantics (no value returned, the thread does not
// wait for it): the executing thread's earlier accesses, and those ordered
// before them by a block barrier, are visible before the add.
__device__ __forceinline__ void red_release_gpu_add(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait of thread 0 of a CTA until *bar >= target (acquire); false and
// the timeout status when the limit runs out.
__device__ __forceinline__ bool spin_until_at_least(const uint32_t *bar, uint32_t target, uint64_t limit_ns,
                                                    uint32_t *status) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
    if (v >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(32);
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
        if (v >= target) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            flag_timeout(status);
            return false;
        }
    }
}

// Barrier of all CTAs of a (cooperatively launched) grid: thread 0 of each CTA
// arrives on *bar and waits (bounded) for `target` arrivals; `flag` is a
// shared word that carries the outcome to the CTA.  Returns false after a
// timeout (recorded in the status word).
__device__ __forceinline__ bool grid_sync(uint32_t *bar, uint32_t target, const BarrierCfg &cfg, uint32_t *status,
                                          uint32_t *flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        // the release arrival covers the CTA's writes (ordered before it by the
        // block barrier); the acquire load of the count covers everyone else's
        red_release_gpu_add(bar, 1u);
        const bool ok = spin_until_at_least(bar, target + cfg.extra, cfg.limit_ns, status);
        *flag = ok ? 1u : 0u;
    }
    __syncthreads();
    return *flag != 0;
}

// Named barrier of `n` threads (whole warps) with id `id` (1..15).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named barrier that also returns, to every participating thread, whether
// `pred` was true in all of them.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Programmatic dependent launch, at the start of every kernel of this
// library: wait until the grid this one was chained after (if it was
// launched as a programmatic dependent) has completed and its memory is
// visible, then allow the next chained grid to be scheduled.  Both are no-ops
// for a kernel launched in plain stream order.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Its two halves, for a kernel that sets up its own shared memory and TMEM
// before it waits: allow the next chained grid to be scheduled ...
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// ... and wait for the grid this one was chained after (before the first
// read of anything that grid may have written).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_inval(uint64_t *bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the completion of the phase with the given parity.
// Returns false (and sets the timeout bit) if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    flag_timeout(status);
    return false;
}

// ------------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// L2 policy for data read exactly once (the streamed key cache): its lines are
// the first to go, so the stream does not push the kernel's code, scores and
// scratch out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Prefetch of the tile at (x, y) of a 2-D tensor map into L2 (no
// destination, nothing to wait for).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                                 int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_1d_hint(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3}], [%2], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "l"(policy)
        : "memory");
}

// Bulk (TMA engine, untiled) copy of `bytes` from global to shared memory,
// completing on `bar` (complete_tx); both addresses 16-byte aligned and bytes
// a multiple of 16.  The barrier's transaction count must cover it
// (mbar_expect_tx or mbar_arrive_expect_tx) before its phase can complete.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Raises the barrier's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Orders this thread's earlier shared-memory accesses (generic proxy) before
// later bulk copies (async proxy) into the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// -------------------------------------------------------------------- tcgen05
// TMEM allocation is warp-collective; the allocated base address is written
// to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzled canonical layout: rows of 128 bytes, 8-row atoms of 1024
// bytes stacked contiguously (stride 1024), base 1024-byte aligned.
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);         // start address
    d |= (uint64_t)1u << 16;                            // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: next 8-row atom
    d |= (uint64_t)1u << 46;                            // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                            // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f8f6f4, A = B = e4m3, K-major both, D = f32.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3_f32(int M, int N) {
    return (1u << 4)                                    // D format f32
           | (0u << 7) | (0u << 10)                     // A, B: e4m3
           | ((uint32_t)(N >> 3) << 17)                 // N / 8
           | ((uint32_t)(M >> 4) << 24);                // M / 16
}

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"   // registers are valid only after the wait
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 bit, one column: this thread's lane of it (warp-collective;
// the lanes are the warp's quarter of TMEM, as in tmem_ld16).
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v)
        : "memory");
}
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r)
        : "r"(taddr)
        : "memory");
    return r;
}

// ------------------------------------------------------------------ misc
// Warp-level histogram increment: lanes with `active` add 1 to hist[bin].
// When every active lane has the same bin (keys that agree on a digit: a
// narrow score range, a radix pass below a common prefix) one atomic adds them
// all; otherwise each lane adds its own (grouping the lanes by bin with
// match.any measured slower for spread bins).  All 32 lanes must call it.
__device__ __forceinline__ void warp_hist_add(uint32_t *hist, uint32_t bin, bool active) {
    const uint32_t amask = __ballot_sync(0xffffffffu, active);
    if (amask == 0) return;
    const uint32_t bmin = __reduce_min_sync(0xffffffffu, active ? bin : 0xFFFFFFFFu);
    const uint32_t bmax = __reduce_max_sync(0xffffffffu, active ? bin : 0u);
    if (bmin == bmax) {
        if ((threadIdx.x & 31) == (uint32_t)(__ffs(amask) - 1)) atomicAdd(&hist[bmin], (uint32_t)__popc(amask));
    } else if (active) {
        atomicAdd(&hist[bin], 1u);
    }
}

// Histogram of the digit (key >> shift) & (nb - 1) of the keys of entries
// j < m whose bits under `mask` equal `prefix`, added into hist by all NT
// threads of the block (warp_hist_add; every warp walks whole 32-entry runs).
// key_at(j, &k) stores entry j's key and returns whether the entry takes part.
template <int NT, class KeyAt>
__device__ __forceinline__ void list_digit_hist(uint32_t *hist, uint32_t m, uint32_t prefix, uint32_t mask, int shift,
                                                uint32_t nb, KeyAt key_at) {
    const uint32_t lane = threadIdx.x & 31u;
    for (uint32_t jb = threadIdx.x & ~31u; jb < m; jb += NT) {
        const uint32_t j = jb + lane;
        uint32_t k = 0u;
        const bool use = j < m && key_at(j, k);
        warp_hist_add(hist, (k >> shift) & (nb - 1), use && (k & mask) == prefix);
    }
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// A relaxed load (no ordering): for polling a flag; follow a hit with
// fence_acq_rel_gpu() before reading what the flag publishes.
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// A 64-bit word that carries its own "published" mark (single-copy atomic):
// no fence is needed to read what it publishes.
__device__ __forceinline__ uint64_t ld_relaxed_gpu_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_gpu_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Atomic add with acquire and release semantics at GPU scope: the caller's
// earlier writes (and those ordered before it by a barrier) are visible to
// whoever acquires the result, and the writes released before the earlier
// adds are visible to the caller.  Returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_release_gpu(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is mapped like +0.0.
__device__ __forceinline__ uint32_t float_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace dsa
