// mbarrier and bulk-copy (TMA, 1-D) helpers for the persistent layer kernel,
// with bounded waits: every wait gives up after a deadline on the global
// timer and reports it, so a kernel never spins forever.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace pmoe {
namespace pipe {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Tests the phase with the given parity; if it is not complete the thread may
// be suspended for a while (a hardware-chosen limit: no time hint is given; a
// 20 us hint and a 100 ns hint measured the same or slightly slower in the
// batch-1 layer) before the test returns false.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete; false if the
// deadline (global timer, ns) passed first. After a few quick tests the thread
// sleeps between tests (up to 256 ns), so that waiting warps leave the issue
// slots to the warps that compute.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t deadline)
{
    uint32_t ns = 16;
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 7) == 0 && globaltimer() > deadline)
            return false;
        if (it >= 2) {
            __nanosleep(ns);
            ns = ns < 256 ? 2 * ns : 256;
        }
    }
}

// The same without sleeping between tests: for hand-overs on a pipeline's critical path (a k-step
// between decoding warps and the MMA thread), where a sleep adds its whole length to the latency;
// the test itself may suspend the thread until the phase completes.
__device__ __forceinline__ bool mbar_wait_tight(uint64_t *bar, uint32_t parity, uint64_t deadline)
{
    for (int it = 0;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 15) == 0 && globaltimer() > deadline)
            return false;
    }
}

// Bulk copy global -> shared (this CTA), completion counted on bar in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Orders this thread's generic-proxy view of global memory (e.g. data another
// CTA released and this thread acquired) before its later bulk copies.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Programmatic dependent launch controls.
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_bar(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

} // namespace pipe
} // namespace pmoe
