// common.cuh -- device helpers shared by the H2O step kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace h2o {

// Error codes a kernel writes into the context's device-visible error word.
enum DeviceError : int {
    kDevOk = 0,
    kDevTimeoutTmaWait = 1,   // a wait for a TMA load ran out of time
    kDevTimeoutMmaWait = 2,   // a wait for a tensor-core commit ran out of time
    kDevTimeoutSlotWait = 3,  // a producer waited too long for a free stage
    kDevTimeoutSelftest = 4,  // the self-test wait (expected to time out)
    kDevBadShape = 5,         // a kernel met a shape it does not handle
};

// Parameters every kernel with a bounded wait receives.
struct WaitBound {
    int* err_word;            // device-visible (host-mapped) error word
    unsigned long long ns;    // give up after this many nanoseconds
};

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(const WaitBound& wb, int code) {
    if (wb.err_word != nullptr) {
        *(volatile int*)wb.err_word = code;
        __threadfence_system();
    }
}

// Programmatic dependent launch: a kernel launched with it may start while
// the previous kernel on the stream is still finishing; it must call
// griddep_wait() before touching global memory that earlier work writes or
// reads. griddep_launch_dependents() lets the next kernel start its own
// prologue early. Both are no-ops for a normal launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return done != 0;
}

// As mbar_try_wait, but the thread may sleep up to `hint_ns` for the phase to
// complete instead of returning at once, so that waiting warps leave the
// issue slots of their SM sub-partition to the warps that compute.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity, uint32_t hint_ns) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(bar_addr), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// Wait until the barrier's phase with the given parity has completed, for at
// most wb.ns nanoseconds. On expiry records `code` and returns false; the
// caller must then stop issuing work and leave.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, const WaitBound& wb,
                                                  int code) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(addr, parity)) return true;
        if (global_ns() - t0 > wb.ns) {
            record_error(wb, code);
            return false;
        }
    }
}

// ---- element conversions ---------------------------------------------------
template <typename E>
__device__ __forceinline__ float to_f32(E x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename E>
__device__ __forceinline__ E from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace h2o
