// ssu_async.cuh -- asynchronous bulk copies and mbarriers for sm_100a (inline PTX).
//
// Used by the streaming kernels to keep several state tiles in flight per warp: the
// Tensor Memory Accelerator's non-tensor bulk copy (cp.async.bulk, global -> shared)
// signals completion on a shared-memory mbarrier through its transaction count. No
// multicast form is used anywhere. Every wait is bounded: after kWaitLimitNs of global
// time it gives up and reports, so a protocol error can never hang the GPU.
//
// Built with SSU_WAIT_TEST (the separate test library libssu_waittest.so, never the
// product libssu.so), the limit comes from a device record that the test sets, and one
// chosen wait can be made to run out: its barrier is armed for 16 bytes more than its
// copies bring, so the copies land but the phase never completes. That exercises every
// give-up path without a fault, a trap or an endless wait.
#pragma once

#include <stdint.h>

#include "ssu_common.cuh"

namespace ssu {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// The bounded waits a test build can make run out.
enum {
    kFaultStream = 1,      // a tile of the per-warp streaming pipeline (decode, replay, ...)
    kFaultPrefill = 2,     // a prefill chunk: its input staging, or (tensor-core form)
                           // its first MMAs, which are then not issued
    kFaultTreeState = 3,   // the tree verify's committed-state rows (tensor-core form)
    kFaultTreeX = 4,       // the tree verify's x tile (tensor-core form)
    kFaultTreeMma = 5      // the tree verify's MMA completion (its MMAs are not issued)
};

#ifdef SSU_WAIT_TEST
// One record per translation unit, set by the test through wait_fault_set_*.
static __device__ WaitFault g_wait_fault = {kWaitLimitNs, 0, -1, -1, -1};

#define SSU_WAIT_FAULT_SETTER(name)                                                        \
    int name(const WaitFault &f)                                                           \
    {                                                                                      \
        return cudaMemcpyToSymbol(g_wait_fault, &f, sizeof f) == cudaSuccess ? 0 : 1;      \
    }
#endif

__device__ __forceinline__ uint64_t wait_limit_ns()
{
#ifdef SSU_WAIT_TEST
    return g_wait_fault.limit_ns;
#else
    return kWaitLimitNs;
#endif
}

// Extra bytes to expect on the barrier of wait `site`, instance `index`, of this CTA's
// warp `warp`: 16 for the one wait a test build was told to make run out, else 0 (always
// 0 in the product build, where this folds away).
__device__ __forceinline__ uint32_t fault_tx(int site, int warp, int index)
{
#ifdef SSU_WAIT_TEST
    const WaitFault &f = g_wait_fault;
    return f.site == site && f.block == (int)blockIdx.x && (f.warp < 0 || f.warp == warp) &&
                   f.index == index
               ? 16u
               : 0u;
#else
    (void)site;
    (void)warp;
    (void)index;
    return 0u;
#endif
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the asynchronous proxy (the bulk-copy unit).
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// A suspend-time hint for the waits (nanoseconds; 0: none), a build-time knob. Measured
// on every kernel with 200 and 1000 ns: within 1 %, so none is given.
#ifndef SSU_WAIT_HINT_NS
#define SSU_WAIT_HINT_NS 0
#endif

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
#if SSU_WAIT_HINT_NS > 0
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"((uint32_t)SSU_WAIT_HINT_NS)
        : "memory");
#else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
#endif
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns(), limit = wait_limit_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 63u) == 0 && global_ns() - t0 > limit)
            return false;
    }
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from global to
// this CTA's shared memory, completing a transaction on `bar`.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace ssu
