// common.cuh -- shared device state and helpers of the MoE layer library.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace moe {

using bf16 = __nv_bfloat16;

// Device-side status word (one per device context).  Kernels record the
// first problem they meet here instead of trapping; the host reads and clears
// it through moe_device_status().  Values are moe_status codes.
__device__ int g_device_status;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

constexpr int kStatusInvalidArg = -1;   // MOE_ERR_INVALID_ARG
constexpr int kStatusTimeout = -4;      // MOE_ERR_TIMEOUT

// Bounded wait on an mbarrier phase.  Returns false (and records a timeout)
// once `timeout_ns` has passed, or at once if another role of the CTA has
// already given up (`abort_flag` set).  After a first plain test the thread
// sleeps in the barrier (suspend-time hint of 20 us) between checks of the
// abort flag and the clock, so a waiting role takes few issue slots.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag, uint64_t timeout_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (abort_flag && *abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > timeout_ns) {
            if (abort_flag) *abort_flag = 1;
            record_status(kStatusTimeout);
            return false;
        }
    }
}

// Warp-wide bounded wait for waits that usually last a whole tile: lane 0
// polls with a short sleep between polls (so the idle warp does not take
// issue slots from the single MMA-issuing thread on the same scheduler),
// then the result is shared with the warp.
__device__ __forceinline__ bool wait_bounded_warp(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag, uint64_t timeout_ns) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        if (!ptx::mbar_try_wait(bar, parity)) {
            const uint64_t t0 = ptx::globaltimer_ns();
            while (true) {
                __nanosleep(256);
                if (ptx::mbar_try_wait(bar, parity)) break;
                if (abort_flag && *abort_flag) {
                    ok = false;
                    break;
                }
                if (ptx::globaltimer_ns() - t0 > timeout_ns) {
                    if (abort_flag) *abort_flag = 1;
                    record_status(kStatusTimeout);
                    ok = false;
                    break;
                }
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

// SiLU for the SwiGLU epilogue, with the fast exponential and division
// intrinsics (the result is rounded to bf16 right after).
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

}  // namespace moe
