// q4k_sm100.cuh -- sm_100a primitives used by the streaming kernels: mbarriers,
// 1-D bulk async copies (TMA, no multicast), named barriers, programmatic
// dependent launch and packed f32x2 FMA. All waits are bounded.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace q4k {

// Fault flag bit raised by a kernel whose bounded wait on a bulk copy gave up.
constexpr unsigned kFaultCopyTimeout = 1u;
// try_wait iterations before a wait is declared lost (each iteration may
// suspend the thread for up to kWaitHintNs, waking early when the phase
// completes), so a lost copy is reported after about a second at most.
constexpr unsigned kSpinLimit = 1u << 20;
constexpr unsigned kWaitHintNs = 1000u;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// One bulk copy global -> shared completing on `bar`. dst, src 16-byte
// aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// One arrival on `bar` (release semantics at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, at most kSpinLimit tries.
// Returns false (and ORs kFaultCopyTimeout into *fault_flags) if it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned* fault_flags) {
    for (unsigned i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
    }
    atomicOr(fault_flags, kFaultCopyTimeout);
    return false;
}

__device__ __forceinline__ void named_barrier_sync(unsigned id, unsigned threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Arrives on named barrier `id` (of `threads` threads) without waiting.
__device__ __forceinline__ void named_barrier_arrive(unsigned id, unsigned threads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch: wait until the preceding grid on the stream
// has completed and its memory is visible / let the next grid start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    return __ffma2_rn(a, b, c);
}

}  // namespace q4k
