// mx_common.cuh -- device-side plumbing shared by the kernels of libmx.so:
// the device error word, bounded waits, and thin inline-PTX wrappers for the
// sm_100a features the kernels use (mbarrier, TMA bulk copies, tcgen05).
//
// Every wait on an mbarrier is bounded by a wall-clock limit (globaltimer);
// when it runs out the waiting thread records MX_DEVERR_TIMEOUT in the error
// word and returns false, and the kernel winds down without touching its
// outputs.  Nothing here traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifndef MX_DEVICE_INLINE
#define MX_DEVICE_INLINE __device__ __forceinline__
#endif

namespace mx {

enum : unsigned { DEVERR_TIMEOUT = 1u, DEVERR_BOUNDS = 2u };

// Site ids recorded with an error (which wait gave up).
enum : unsigned {
    SITE_GEMM_PRODUCER_EMPTY = 1,
    SITE_GEMM_MMA_FULL = 2,
    SITE_GEMM_EPI_ACC = 3,
    SITE_GEMM_MMA_ACC_EMPTY = 4,
    SITE_GEMM_TAIL = 5,
    SITE_FUSED_PRODUCER_EMPTY = 6,
    SITE_GEMM_EPI_DRAIN = 7,
    SITE_GEMM_SF_FULL = 8,
    SITE_GEMM_SF_EMPTY = 9,
    SITE_GEMM_MMA_SF = 10,
    SITE_GEMM_SF_LOAD = 11,
    SITE_GEMM_SF_FREE = 12,
    SITE_GEMM_MMA_READY = 13,
    SITE_FUSED_BAND_READY = 14,   // a TMA producer waiting for a band of the fused quantize
    SITE_KSPLIT_PARTIAL = 15,     // a finishing piece waiting for the partial sums of its tile
};

// {flags, first site, first block, count}
__device__ unsigned int g_error_word[4];

MX_DEVICE_INLINE void record_error(unsigned flag, unsigned site) {
    atomicOr(&g_error_word[0], flag);
    if (atomicCAS(&g_error_word[1], 0u, site) == 0u) g_error_word[2] = blockIdx.x + 65536u * blockIdx.y;
    atomicAdd(&g_error_word[3], 1u);
}

MX_DEVICE_INLINE uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

MX_DEVICE_INLINE uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
MX_DEVICE_INLINE void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

MX_DEVICE_INLINE void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

MX_DEVICE_INLINE void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

MX_DEVICE_INLINE void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

MX_DEVICE_INLINE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

MX_DEVICE_INLINE bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}



// Wait for the phase with the given parity to complete, for at most limit_ns.
// Returns false (and records a timeout) if it did not, or if *abort is set by
// another role of the same CTA that already gave up.
MX_DEVICE_INLINE bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns, unsigned site,
                                        volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 0u) {
            if (abort != nullptr && *abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                record_error(DEVERR_TIMEOUT, site);
                if (abort != nullptr) *abort = 1;
                return false;
            }
        }
    }
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running; griddep_wait() returns once that kernel has completed and its
// memory is visible, so everything before it must not read the previous
// kernel's outputs.  griddep_launch_dependents() lets the next such kernel be
// scheduled early (it still waits for this one's completion in its own
// griddep_wait()).  Both are no-ops for kernels launched without the attribute.
MX_DEVICE_INLINE void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MX_DEVICE_INLINE void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// A shared-memory counter published by one warp (release) and polled by
// another (acquire): cheaper to read than an mbarrier when the reader only
// needs to know how far the writer has got.
MX_DEVICE_INLINE void st_release_shared(uint32_t *p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
MX_DEVICE_INLINE uint32_t ld_acquire_shared(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Poll *counter until it exceeds `need` (bounded like the mbarrier waits).
// Returns the value seen, or 0 after recording a timeout.
MX_DEVICE_INLINE uint32_t wait_counter_above(const uint32_t *counter, uint32_t need, uint64_t limit_ns, unsigned site,
                                             volatile int *abort) {
    uint32_t v = ld_acquire_shared(counter);
    if (v > need) return v;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        v = ld_acquire_shared(counter);
        if (v > need) return v;
        if ((i & 15u) == 0u) {
            if (abort != nullptr && *abort) return 0u;
            if (globaltimer_ns() - t0 > limit_ns) {
                record_error(DEVERR_TIMEOUT, site);
                if (abort != nullptr) *abort = 1;
                return 0u;
            }
        }
    }
}

// ---------------------------------------------------------------- cross-CTA counters
// A global counter advanced by the CTAs that produce data (release at gpu scope)
// and polled by the CTAs that consume it (acquire at gpu scope).  The consumers
// read the data with TMA, i.e. through the async proxy: the producer orders its
// ordinary stores before the release with fence.proxy.async.global, and the
// consumer orders its TMA loads after the acquire with another one.
MX_DEVICE_INLINE void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
MX_DEVICE_INLINE uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
MX_DEVICE_INLINE void red_release_gpu_add(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Poll *counter until it reaches target (bounded like the mbarrier waits), then
// order the caller's later async-proxy (TMA) reads after what it observed.
MX_DEVICE_INLINE bool wait_global_at_least(const uint32_t *counter, uint32_t target, uint64_t limit_ns, unsigned site,
                                           volatile int *abort) {
    if (ld_acquire_gpu(counter) < target) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = 1;; ++i) {
            __nanosleep(64);
            if (ld_acquire_gpu(counter) >= target) break;
            if ((i & 7u) == 0u) {
                if (abort != nullptr && *abort) return false;
                if (globaltimer_ns() - t0 > limit_ns) {
                    record_error(DEVERR_TIMEOUT, site);
                    if (abort != nullptr) *abort = 1;
                    return false;
                }
            }
        }
    }
    fence_proxy_async_global();
    return true;
}

// Barrier over the 128 threads of warps 2-5 of a GEMM CTA (hardware barrier 1;
// barrier 0 is __syncthreads).
MX_DEVICE_INLINE void sync_epilogue_warps() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// ---------------------------------------------------------------- packed fp32 pairs
// f32x2 arithmetic of sm_100: two IEEE operations per instruction, each
// rounded exactly as its scalar form (nearest-even, or toward zero for mul2_rz).
MX_DEVICE_INLINE uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
MX_DEVICE_INLINE void upk2(uint64_t r, float &a, float &b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r)); }
MX_DEVICE_INLINE uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
MX_DEVICE_INLINE uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
MX_DEVICE_INLINE uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
MX_DEVICE_INLINE uint64_t mul2_rz(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
MX_DEVICE_INLINE uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// ---------------------------------------------------------------- TMA / bulk copies
MX_DEVICE_INLINE void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2D tiled TMA load (no multicast) into this CTA's shared memory.
MX_DEVICE_INLINE void tma_load_2d(void *smem_dst, const void *tmap, int32_t x, int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Untiled bulk copy (no multicast) of `bytes` from global memory into this
// CTA's shared memory; both addresses 16-byte aligned, bytes a multiple of 16.
MX_DEVICE_INLINE void bulk_load(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 3D tiled TMA load (no multicast) into this CTA's shared memory.
MX_DEVICE_INLINE void tma_load_3d(void *smem_dst, const void *tmap, int32_t x, int32_t y, int32_t z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}



// 2D tiled TMA store (bulk-group completion) from this CTA's shared memory.
MX_DEVICE_INLINE void tma_store_2d(const void *tmap, int32_t x, int32_t y, const void *smem_src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(x), "r"(y), "r"(smem_u32(smem_src))
                 : "memory");
}
MX_DEVICE_INLINE void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read shared memory.
template <int N>
MX_DEVICE_INLINE void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all committed bulk groups have completed (writes performed).
MX_DEVICE_INLINE void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05
MX_DEVICE_INLINE void tmem_alloc(uint32_t *smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
MX_DEVICE_INLINE void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MX_DEVICE_INLINE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
MX_DEVICE_INLINE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MX_DEVICE_INLINE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }



// Block-scaled MMAs: D(tmem) (+)= (A * sfA) x (B * sfB)^T, A/B described in smem.
MX_DEVICE_INLINE void tc_mma_mxf8f6f4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                      uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
MX_DEVICE_INLINE void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                  uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
MX_DEVICE_INLINE void tc_mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                  uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one row per thread).
MX_DEVICE_INLINE void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
MX_DEVICE_INLINE void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
MX_DEVICE_INLINE void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Store 16 consecutive 32-bit TMEM columns of this warp's 32 lanes (one register
// per lane and column), then wait for the stores to complete.
MX_DEVICE_INLINE void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
MX_DEVICE_INLINE void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
MX_DEVICE_INLINE void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
MX_DEVICE_INLINE void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// ---------------------------------------------------------------- clusters (CTA pairs)
MX_DEVICE_INLINE uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
MX_DEVICE_INLINE void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of this cluster.
MX_DEVICE_INLINE uint32_t mapa_shared(uint32_t local_saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_saddr), "r"(rank));
    return r;
}
// Arrive (relaxed, cluster scope) on an mbarrier given by its shared::cluster
// address.  Callers order their tcgen05 stores before it with tcgen05.wait::st
// and tcgen05.fence::before_thread_sync; a release at cluster scope costs
// about a thousand cycles per arrive here and is not needed for that order.
MX_DEVICE_INLINE void mbar_arrive_cluster(uint32_t cluster_saddr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_saddr) : "memory");
}
// 2D tiled TMA load into this CTA's shared memory whose completion is signalled
// on an mbarrier of the pair's leader CTA (cta_group::2 form, no multicast).
MX_DEVICE_INLINE void tma_load_2d_pair(void *smem_dst, const void *tmap, int32_t x, int32_t y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
MX_DEVICE_INLINE void tmem_alloc_pair(uint32_t *smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
MX_DEVICE_INLINE void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MX_DEVICE_INLINE void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive on the mbarrier at this offset in every CTA of `cta_mask` once all prior
// tcgen05 operations of this thread (issued for the CTA pair) complete.
MX_DEVICE_INLINE void tc_commit_pair(uint64_t *bar, uint16_t cta_mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"(cta_mask)
                 : "memory");
}
// Block-scaled MMAs of a CTA pair (M = 256 across the two CTAs' TMEM).
MX_DEVICE_INLINE void tc_mma_pair_mxf8f6f4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                           uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
MX_DEVICE_INLINE void tc_mma_pair_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
MX_DEVICE_INLINE void tc_mma_pair_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}


// ---------------------------------------------------------------- predicated tcgen05 issue
// The whole warp executes these with warp-uniform operands; only threads whose
// `issue` flag is set perform the operation.  (No branch: operands stay uniform.)
MX_DEVICE_INLINE void tc_commit_if(uint64_t *bar, uint32_t issue) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar)),
        "r"(issue)
        : "memory");
}
MX_DEVICE_INLINE void tc_commit_pair_if(uint64_t *bar, uint16_t cta_mask, uint32_t issue) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t"
        "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask), "r"(issue)
        : "memory");
}
#define MX_DEFINE_MMA_IF(NAME, GROUP, KIND)                                                                        \
    MX_DEVICE_INLINE void NAME(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,          \
                               uint32_t sfb, uint32_t accumulate, uint32_t issue) {                                 \
        asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 q, %7, 0;\n\t"                   \
                     "@q tcgen05.mma.cta_group::" GROUP ".kind::" KIND " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d), \
                     "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb), "r"(issue)             \
                     : "memory");                                                                                   \
    }
MX_DEFINE_MMA_IF(tc_mma_mxf8f6f4_if, "1", "mxf8f6f4.block_scale")
MX_DEFINE_MMA_IF(tc_mma_mxf4_if, "1", "mxf4.block_scale.block32")
MX_DEFINE_MMA_IF(tc_mma_nvf4_if, "1", "mxf4nvf4.block_scale.block16")
MX_DEFINE_MMA_IF(tc_mma_pair_mxf8f6f4_if, "2", "mxf8f6f4.block_scale")
MX_DEFINE_MMA_IF(tc_mma_pair_mxf4_if, "2", "mxf4.block_scale.block32")
MX_DEFINE_MMA_IF(tc_mma_pair_nvf4_if, "2", "mxf4nvf4.block_scale.block16")
#undef MX_DEFINE_MMA_IF

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (sm_100 form): start >> 4 in bits [0,14),
// leading byte offset >> 4 in [16,30), stride byte offset >> 4 in [32,46),
// version 1 in [46,48), layout type in [61,64) (0 none, 2 = 128-byte swizzle).
MX_DEVICE_INLINE uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}


}  // namespace mx
