// tma.cuh -- tensor-memory-accelerator loads and mbarrier waits for sm_100a.
//
// The sequence kernels read channel-last [B, L, D] tiles that are only a few
// channels wide: every time step of a tile is a separate 16..32-byte piece of
// global memory.  Issuing those pieces from the threads costs one load-store
// request per piece and stalls the issuing warps behind the memory pipeline;
// a TMA box [t: up to 256][d: ROWS] is one instruction from one thread, the
// address generation and the zero fill past the tensor's edges (t >= L, the
// transform's padding, and d >= D, a ragged last channel group) happen in the
// copy engine, and completion is counted in bytes on an mbarrier.
//
// Every wait is bounded in time: a wait that runs out sets a bit in the
// per-device fault word (read by causal_conv_fault_flags) and the kernel
// returns instead of hanging.  No load here uses cluster multicast.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ccv {

// Fault bits, or-ed into g_cc_fault by kernels whose bounded waits ran out.
constexpr unsigned kFaultTmaWait = 1u;
__device__ unsigned int g_cc_fault;

// Wait limit: two seconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    // make the initialised barrier visible to the copy engine
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and announce `bytes` of incoming transactions for this phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Named barrier over `count` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

// Named barrier over `count` threads that also and-reduces `pred` across them.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
    unsigned r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((unsigned)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// Arrive once (no transaction count).
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after the time limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// Order this thread's earlier generic-proxy shared-memory accesses (made
// visible to it by a CTA barrier) before later async-proxy writes.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 3-D tiled TMA load of one box into shared memory, completing on `bar`.
// x (innermost) * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace ccv
