// watchdog.cuh -- bounded waits on shared-memory mbarriers.
//
// Every wait in libosdn polls a bounded number of times.  When the bound runs out the
// waiting thread records OSDN_ERR_DEVICE_TIMEOUT in the device status word and reports
// failure to its caller, which then leaves the kernel in an orderly way; no kernel traps or
// spins forever.
#pragma once

#include "common.cuh"

namespace osdn {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The dynamic shared-memory buffer advanced to a 1024-byte boundary by pointer arithmetic on the
// __shared__ array itself, so the compiler still knows the result points to shared memory (a
// round trip through an integer type would leave it a generic pointer: slower accesses that it
// must also keep in order with global stores).
__device__ __forceinline__ uint8_t* smem_align1024(uint8_t* raw) {
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test_parity(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_try_parity(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait until the phase with the given parity has completed, for at most `limit_ns`
// nanoseconds of wall time.  Returns false (after recording OSDN_ERR_DEVICE_TIMEOUT) if it
// never completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  int64_t limit_ns) {
    if (mbar_try_parity(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_parity(bar, parity)) return true;
        if (global_ns() - t0 > static_cast<uint64_t>(limit_ns)) break;
    }
    record_status(OSDN_ERR_DEVICE_TIMEOUT);
    return false;
}

// Bound on every wait inside the tensor-core kernels: far above any legitimate wait (those
// last microseconds), short enough that a stuck kernel returns within seconds.
constexpr int64_t kWaitLimitNs = 2000000000LL;

// Diagnostic kernel: waits on a barrier that nobody arrives at, with a bounded number of
// non-blocking polls, so that the timeout path runs and the kernel returns.
__global__ void watchdog_selftest_kernel(int64_t spin_limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar, 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        bool done = false;
        for (int64_t i = 0; i < spin_limit && !done; ++i) done = mbar_test_parity(&bar, 0);
        if (!done) record_status(OSDN_ERR_DEVICE_TIMEOUT);
    }
    __syncthreads();
}

}  // namespace osdn
