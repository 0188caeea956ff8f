// sm_100a asynchronous-copy, mbarrier and cluster primitives (inline PTX), and
// the host-side tensor-map encoder.
//
// Every wait is bounded: after kWaitCycles of polling it records
// NVFP4_ERR_DEVICE_TIMEOUT in the library status word and returns false, so a
// kernel whose producer never delivers exits instead of hanging the GPU.
// No load here uses cluster multicast: every CTA fetches its own tiles.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace nvfp4 {

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz

NVFP4_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel before it in the stream is still
// running.  griddep_wait() returns once that kernel has completed and its
// writes are visible; nothing an earlier kernel may still be writing (the
// activations) is read, and no output is written, before it.  Weights are
// read-only for the duration of a forward pass and may be fetched before it.
// griddep_launch_dependents() lets the next such kernel start as soon as every
// CTA of this grid has issued it.
NVFP4_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
NVFP4_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

NVFP4_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
NVFP4_DEV void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
NVFP4_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

NVFP4_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
NVFP4_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Release a slot after reading it with ordinary shared-memory loads.  The
// arrive takes `dep` (a value computed from everything read out of the slot)
// as an input, so it cannot issue before those loads have returned their
// data; a plain arrive can overtake loads still in flight, and the producer's
// next copy into the slot would then race them.
NVFP4_DEV void mbar_arrive_after(uint64_t* bar, uint32_t dep) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)), "r"(dep) : "memory");
}
// Warp-wide release of a slot: `dep` folds every word this lane read from the
// slot; the butterfly makes lane 0's copy depend on all 32 lanes' reads, and
// lane 0 alone arrives (barrier count: one per warp).
NVFP4_DEV void warp_release_after(uint64_t* bar, uint32_t dep) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dep ^= __shfl_xor_sync(0xffffffffu, dep, o);
    if ((threadIdx.x & 31) == 0) mbar_arrive_after(bar, dep);
}
NVFP4_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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
// Bounded wait for the phase with the given parity to complete: false (and
// NVFP4_ERR_DEVICE_TIMEOUT recorded in *status) after `limit` cycles.
NVFP4_DEV bool mbar_wait_limit(uint64_t* bar, uint32_t parity, int* status, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            if (status) atomicExch(status, NVFP4_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}
NVFP4_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
    return mbar_wait_limit(bar, parity, status, kWaitCycles);
}

// 2D tiled TMA load (no multicast) completing on `bar`.
NVFP4_DEV void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// 1D bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0).
NVFP4_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// L2 policy for data read once (streamed weights): evicted first, so that it
// does not push out activations, outputs and workspace.
NVFP4_DEV uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
NVFP4_DEV void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
NVFP4_DEV void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
NVFP4_DEV void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---- clusters ------------------------------------------------------------
NVFP4_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
NVFP4_DEV void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Split cluster barrier: arrive early (relaxed: orders nothing), wait later.
NVFP4_DEV void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
NVFP4_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
// Store a float to the same shared-memory offset in CTA `rank` of the cluster.
NVFP4_DEV void st_dsmem_f32(float* local, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
// Read a float from the same shared-memory offset in CTA `rank` of the cluster.
NVFP4_DEV float ld_dsmem_f32(const float* local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// ---- host: tensor maps -------------------------------------------------------
// 2D row-major byte matrix [rows, row_bytes] (row stride = row_bytes), box of
// box_bytes x box_rows, no swizzle, out-of-bounds elements read as zero.
bool make_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes,
                     uint32_t box_rows, int swizzle128 = 0);

}  // namespace nvfp4
