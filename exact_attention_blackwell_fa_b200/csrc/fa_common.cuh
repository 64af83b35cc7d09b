// fa_common.cuh -- pieces shared by the forward and backward kernels: device status
// word, bounded mbarrier waits, 16-bit packing, the split MUFU / FMA-polynomial exp2.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/fa.h"
#include "exp2_poly.h"
#include "sm100.cuh"

namespace fa {

// Every wait in the kernels gives up after this long and reports FA_ERR_DEVICE_TIMEOUT.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;

// Device status: [0] fa_status code of the first failure, [1] code of the wait that
// gave up, [2] block index, [3] unused.
__device__ uint32_t g_status[4];

// Per-CTA control block in shared memory.
struct CtaCtl {
    uint32_t tmem_base;
    uint32_t abort;  // set when any wait of this CTA gave up; other waits then bail out
};

__device__ __forceinline__ void record_timeout(uint32_t where)
{
    if (atomicCAS(&g_status[0], 0u, static_cast<uint32_t>(FA_ERR_DEVICE_TIMEOUT)) == 0u) {
        g_status[1] = where;
        g_status[2] = blockIdx.x;
    }
}

// Single-thread bounded wait.  Returns false (and raises the CTA abort flag) if the
// phase did not complete within kWaitTimeoutNs, or if another wait already aborted.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, CtaCtl* ctl, uint32_t where)
{
    if (mbar_try_wait(bar, parity)) return true;
    volatile uint32_t* abort = &ctl->abort;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > kWaitTimeoutNs) {
                *abort = 1u;
                record_timeout(where);
                return false;
            }
        }
    }
}

// Bounded wait that ignores the abort flag: used while draining in-flight copies or
// MMAs before the CTA exits, which always complete on their own.
__device__ __noinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint32_t where)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            record_timeout(where);
            return false;
        }
    }
    return true;
}

// Warp-wide wait: lane 0 polls, the result is broadcast (the shuffle also syncs the warp).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, CtaCtl* ctl,
                                          uint32_t where)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, ctl, where) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ---------------------------------------------------------------------------------
// 16-bit packing: two fp32 values -> one 32-bit word, `lo` in the low half.
// ---------------------------------------------------------------------------------
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&w);
        return __bfloat1622float2(v);
    } else {
        __half2 v = *reinterpret_cast<__half2*>(&w);
        return __half22float2(v);
    }
}

// ---------------------------------------------------------------------------------
// 2^x on the FMA pipe (x <= 8 in use): x = n + f, n = round(x), f in [-1/2, 1/2];
// p(f) is our own relative-minimax cubic (exp2_poly.h); 2^n is applied by adding n to
// the exponent field.  x is clamped at -126 so the exponent add cannot wrap.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float exp2_fma(float x)
{
    x = fmaxf(x, -126.0f);
    const float shifter = 12582912.0f;  // 1.5 * 2^23: adding it rounds x to an integer
    const float t = __fadd_rn(x, shifter);
    const float n = __fsub_rn(t, shifter);
    const float f = __fsub_rn(x, n);
    float p = fmaf(FA_EXP2_C3, f, FA_EXP2_C2);
    p = fmaf(p, f, FA_EXP2_C1);
    p = fmaf(p, f, FA_EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace fa
