// Device helpers shared by the W8A16 kernels: mbarrier and TMA wrappers,
// tcgen05 (5th-generation tensor core / tensor memory) wrappers, bounded
// waits, the device status word and int8 -> fp16 widening.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace w8 {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ---------------------------------------------------------------- status
// Status word of this module on each device: 0 = fine; otherwise bit 0 set
// and bits 8..15 hold the site of the first wait that ran out.
__device__ unsigned int g_status;

enum WaitSite : unsigned {
    SITE_Q_LOAD = 0x10,
    SITE_Q_EMPTY = 0x11,
    SITE_Q_XCHG = 0x12,
    SITE_Q_SYNC = 0x13,
    SITE_DEC_EMPTY = 0x20,
    SITE_DEC_FULL = 0x21,
    SITE_DEC_FIX = 0x22,
    SITE_DEC_DRAIN = 0x23,
    SITE_DEC_PUB = 0x24,     // helper: the consumers' first part stored
    SITE_DEC_START = 0x25,   // consumers: the helper's count of that part
    SITE_DEC_PRE = 0x26,     // consumers: the helper's look at the next CTA's part
    SITE_DEC_POLL = 0x27,    // helper: polling for the next CTA's part
    SITE_DEC_CLUSTER = 0x28, // cluster split: the peers' parts in CTA 0
    SITE_PF_EMPTY = 0x30,
    SITE_PF_FULL_CVT = 0x31,
    SITE_PF_FULL_MMA = 0x32,
    SITE_PF_AEMPTY = 0x33,
    SITE_PF_AFULL = 0x34,
    SITE_PF_DEMPTY = 0x35,
    SITE_PF_DFULL = 0x36,
    SITE_PF_DRAIN = 0x37,
    SITE_PF_XEMPTY = 0x38,
    SITE_P2_WEMPTY = 0x40,
    SITE_P2_XEMPTY = 0x41,
    SITE_P2_WFULL = 0x42,
    SITE_P2_XFULL = 0x43,
    SITE_P2_AEMPTY = 0x44,
    SITE_P2_AFULL = 0x45,
    SITE_P2_DEMPTY = 0x46,
    SITE_P2_DFULL = 0x47,
    SITE_P2_DRAIN = 0x48,
    SITE_P2_FIX = 0x49,
    SITE_CLIP_EMPTY = 0x50,
    SITE_CLIP_LOAD = 0x51,
    SITE_CLIP_DRAIN = 0x52,
    SITE_SELFTEST = 0xEE,
};

// One second: every legitimate wait in these kernels lasts microseconds.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ void record_timeout(unsigned site) {
    atomicCAS(&g_status, 0u, (site << 8) | 1u);
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- programmatic dependent launch
// Let the next kernel in the stream (launched with programmatic stream
// serialization) start its prologue while this grid is still running.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the previous grid in the stream has completed and its memory
// operations are visible (returns at once when there is none).
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Bring [src, src + bytes) into L2 without touching shared memory (16-byte
// aligned address, size a multiple of 16).  Safe before pdl_wait: L2 is
// coherent, so a later write by the previous grid simply updates the lines.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- global memory ordering
// Load with acquire semantics at GPU scope.
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Atomic add at GPU scope with acquire-release semantics: publishes what
// this thread (and, through a preceding CTA barrier, its CTA) wrote before
// it, and orders what it reads after it.
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// ---------------------------------------------------------------- smem
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of a phase (acquire at CTA scope when it reports
// completion).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may park the thread (without issuing) for up to `hint_ns`
// until the phase completes, instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for waiters that should not take issue slots from the
// threads doing the work (many warps waiting on one barrier): each try
// parks the thread for up to 20 us.
__device__ __forceinline__ bool mbar_wait_parked(uint64_t *bar, uint32_t parity, unsigned site,
                                                 unsigned long long limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i) {
            if (mbar_try_wait_sleep(a, parity, 20000u)) return true;
        }
        if (globaltimer_ns() - t0 > limit_ns) {
            record_timeout(site);
            return false;
        }
    }
}

// Wait until the barrier's phase with the given parity has completed.
// Gives up after `limit_ns`, records `site` and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned site,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    // the clock is read only once a wait is long (it costs time in the
    // streaming loops, where almost every wait ends within these tries)
#pragma unroll 1
    for (int i = 0; i < 512; ++i) {
        if (mbar_try_wait(a, parity)) return true;
    }
    const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 512; ++i) {
            if (mbar_try_wait(a, parity)) return true;
        }
        if (globaltimer_ns() - t0 > limit_ns) {
            record_timeout(site);
            return false;
        }
    }
}

// The same decision in every lane of the warp (all lanes must call it):
// after a bounded wait, lanes whose waits ended differently would otherwise
// diverge before warp-collective instructions.
__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok) != 0; }

// ---------------------------------------------------------------- TMA
// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Same with an L2 eviction-priority policy (createpolicy result).
__device__ __forceinline__ void bulk_g2s_hint(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled tensor load (box given by the tensor map) at element
// coordinates (x = innermost, y).  x * element size must be a multiple of
// 16 bytes; out-of-range elements are filled with zero.
__device__ __forceinline__ void tma_load_3d(void *dst_smem, const CUtensorMap *map, int32_t x, int32_t y,
                                            int32_t z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst_smem, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Same with an L2 eviction-priority policy (createpolicy result).
__device__ __forceinline__ void tma_load_2d_hint(void *dst_smem, const CUtensorMap *map, int32_t x,
                                                 int32_t y, uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
    return v;
}
// Asynchronous store of four floats (16-byte aligned) into the shared
// memory of some CTA of the cluster; its 16 bytes are counted (complete_tx)
// on that CTA's mbarrier `cluster_bar`, whose phase completes once every
// expected byte has landed, with no fence on the storing side.
__device__ __forceinline__ void st_async_dsmem_v4(uint32_t cluster_addr, float a, float b, float c, float d,
                                                  uint32_t cluster_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     cluster_addr),
                 "f"(a), "f"(b), "f"(c), "f"(d), "r"(cluster_bar)
                 : "memory");
}
// Split cluster barrier: every thread of the cluster arrives once (relaxed:
// the writes to publish are fenced separately, e.g. by
// fence.mbarrier_init), and a thread that will touch another CTA's shared
// memory waits for the phase first.  Whole warps (.aligned).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    __syncwarp();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
// Arrive once on an mbarrier of some CTA of the cluster, releasing this
// thread's prior writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// Arrive once on an mbarrier of some CTA of the cluster with the default
// (CTA-scope) semantics.  For signals whose data is ordered by other means
// -- tensor-memory stores and loads completed with tcgen05.wait and fenced
// with tcgen05.fence::before_thread_sync -- this avoids the cost of a
// cluster-scope release (about a microsecond per arrive).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar_addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on a local barrier whose arrivals come from the whole
// cluster (acquire at cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, unsigned site,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
#pragma unroll 1
    for (int i = 0; i < 512; ++i) {
        if (mbar_try_wait_acq_cluster(a, parity)) return true;
    }
    const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 512; ++i) {
            if (mbar_try_wait_acq_cluster(a, parity)) return true;
        }
        if (globaltimer_ns() - t0 > limit_ns) {
            record_timeout(site);
            return false;
        }
    }
}
// Full cluster barrier (every thread of every CTA of the cluster).
// All threads of the cluster (the .aligned forms need whole warps: a warp
// whose lanes took different paths meets here first).
__device__ __forceinline__ void cluster_sync_all() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// 2-D tensor load into this CTA's shared memory whose completion is
// counted on `bar_cluster`, an mbarrier of either CTA of the pair
// (shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void *dst_smem, const CUtensorMap *map, int32_t x,
                                                 int32_t y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// D[tmem, both CTAs] (+)= A[tmem, both CTAs] * B[smem desc, both CTAs]:
// M = 256 (128 rows in each CTA), issued by one thread of the pair's
// first CTA.
__device__ __forceinline__ void tc_mma_ts_f16_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                   uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at `bar`'s offset in each CTA of `cta_mask`
// when all prior pair MMAs of this thread have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over nthreads threads that also returns whether pred holds in
// all of them (so that a group of warps agrees on giving up a wait).
__device__ __forceinline__ bool named_bar_all(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------- int8 widening
// A byte u = q + 128 (offset binary) placed under the fp16 exponent pattern
// 0x64 encodes 1024 + u exactly; subtracting 1152 = 1024 + 128 leaves q.
// prmt selects bytes 0,1 (or 2,3) of `w` into the low byte of each half.
__device__ __forceinline__ uint32_t widen_lo2(uint32_t w) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x64646464u), "r"(0x4140u));
    return r;
}
__device__ __forceinline__ uint32_t widen_hi2(uint32_t w) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x64646464u), "r"(0x4342u));
    return r;
}
// fp16x2 subtraction of (1152, 1152); exact for the values produced above.
__device__ __forceinline__ uint32_t unbias2(uint32_t h2) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h2), "r"(0x64806480u));
    return r;
}
// With a zero point z (asymmetric codes): the pair minus (1152 + z), i.e.
// the codes q - z, exact (|q - z| <= 255).  c = zp_bias2(z).
__device__ __forceinline__ uint32_t unbias2_by(uint32_t h2, uint32_t c) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h2), "r"(c));
    return r;
}
// fp16 1152 + z in both halves: for z in [-128, 127] the value lies in
// [1024, 1279], where the fp16 pattern is 0x6400 plus (value - 1024).
__device__ __forceinline__ uint32_t zp_bias2(int z) {
    const uint32_t h = 0x6480u + (uint32_t)z;
    return h | (h << 16);
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
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
// Arrive once on `bar` when all previously issued tcgen05.mma of this
// thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (fp16 inputs, fp32 accum).
__device__ __forceinline__ void tc_mma_ts_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}


// Store 32 consecutive 32-bit columns of this thread's TMEM lane.
// Store 32 columns of this warp's 32 lanes and wait until the store has
// read them, in ONE asm statement.  tcgen05.st reads its source registers
// asynchronously, until tcgen05.wait::st; with the wait in a later statement
// the compiler takes the registers as free once the store is issued and may
// reuse them for the next values first (seen here as 32 channels of a tile
// widened wrongly, depending on the instantiation's register allocation).
__device__ __forceinline__ void tmem_store_32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Load 32 consecutive 32-bit columns of this thread's TMEM lane.

// Load 32 columns of this warp's 32 lanes and wait for them, in ONE asm
// statement.  tcgen05.ld writes its registers asynchronously: until
// tcgen05.wait::ld they hold no data.  With the two in separate statements
// the compiler treats the registers as valid right after the load and, under
// register pressure, may spill them in between -- saving values that have not
// arrived (seen here as whole warps of wrong outputs).  One statement leaves
// it no point to do so.
__device__ __forceinline__ void tmem_load_32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by a
// TMA load with 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes
// apart.  Fields: start address >> 4 (bits 0-13), leading byte offset >> 4
// (16-29, unused for swizzled K-major; 1), stride byte offset >> 4
// (32-45), descriptor version 1 (46-47), layout type 2 = 128B swizzle
// (61-63).
__device__ __forceinline__ uint64_t smem_desc_kmajor_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor for kind::f16: fp16 A and B, fp32 accumulator,
// both operands K-major, shape M x N.  Fields: c_format (bits 4-5) = 1
// (F32), a_format (7-9) = 0 (F16), b_format (10-12) = 0 (F16), a/b major
// (15, 16) = 0 (K), N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t m, uint32_t n) {
    return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

}  // namespace w8
