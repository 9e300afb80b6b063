// common.cuh -- status reporting and bounded waits shared by the kernels.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "attn.h"
#include "ptx.cuh"

namespace attn {

// Device-side status word, read and cleared by attn_get_device_status().
// The first non-OK code reported since the last read wins.
__device__ int g_attn_status = 0;

__device__ __forceinline__ void report_status(int code) { atomicCAS(&g_attn_status, 0, code); }

// A wait on an mbarrier gives up after this many SM cycles (about a second at the
// clocks a B200 runs): no legitimate wait in these kernels comes anywhere near it.
constexpr long long kWaitLimitCycles = 2000000000LL;
// Waits that only drain work already in flight after an abort use a shorter bound.
constexpr long long kDrainLimitCycles = 200000000LL;

// Bounded wait for the phase `parity` of `bar`. Returns false if this CTA gave up:
// either this wait ran out (it then raises the CTA's abort flag and reports
// ATTN_ERR_TIMEOUT) or another role of the CTA already raised the abort flag.
// Never traps and never spins without a limit.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity,
                                           volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitLimitCycles) {
            *abort_flag = 1;
            report_status(ATTN_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait used only while draining after an abort; ignores the abort flag.
__device__ __forceinline__ void drain_phase(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kDrainLimitCycles) return;
    }
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if constexpr (BF16) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&w);
        return __bfloat1622float2(v);
    } else {
        __half2 v = *reinterpret_cast<__half2*>(&w);
        return __half22float2(v);
    }
}

constexpr int kPageSize = 16;  // tokens per block of a paged KV cache

// Mask modes, fixed at compile time so the common cases carry no window arithmetic.
enum : int { kMaskNone = 0, kMaskCausal = 1, kMaskWindow = 2 };

constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

}  // namespace attn
