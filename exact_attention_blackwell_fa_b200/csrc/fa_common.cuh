// fa_common.cuh -- pieces shared by the forward and backward kernels: device status
// word, bounded mbarrier waits, 16-bit packing, the split MUFU / FMA-polynomial exp2.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/fa.h"
#include "exp2_poly.h"
#include "sm100.cuh"

namespace fa {

// Every pipeline wait in the kernels gives up after CtaCtl::wait_ns (the launch's
// setting, fa_set_wait_timeout_ms; this by default) and reports FA_ERR_DEVICE_TIMEOUT.
// The limit is wall-clock time (%globaltimer), which keeps running while the GPU
// serves another context, so a time slice longer than the limit reads as a timeout.
// Drains -- waits for copies and MMAs already issued, which always complete -- allow
// at least this much whatever the setting.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;
// Spinning waits (SPIN below) first poll without suspending (test_wait) for this many
// probes, then fall back to the suspending, timed loop: a thread suspended in try_wait
// was measured to resume hundreds of cycles after the phase completed, which costs a
// pipeline whose step time is made of such hand-offs; the polls in turn take issue
// slots from the warps they share a scheduler with, so each kernel chooses.
constexpr uint32_t kSpinPolls = 1u << 16;

// Device status: [0] fa_status code of the first failure, [1] code of the wait that
// gave up, [2] block index, [3] unused.
__device__ uint32_t g_status[4];

// Per-CTA control block in shared memory.
struct CtaCtl {
    uint32_t tmem_base;
    uint32_t abort;    // set when any wait of this CTA gave up; other waits then bail out
    uint64_t wait_ns;  // limit of a pipeline wait, from the launch parameters
};

// Unit of round r of a persistent CTA's static walk: rounds take gridDim.x consecutive
// units, CTA b the b-th of an even round and the b-th from the end of an odd one.
// With the unit list sorted longest first (causal), a CTA that took a long unit of a
// round takes a short one of the next, so the CTAs' totals stay level; each round is
// a permutation of the plain stride's, so every unit below the count is walked once
// and the first index past the count ends the walk.
__device__ __forceinline__ int walk_unit(int r)
{
    const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    return r * g + ((r & 1) ? g - 1 - b : b);
}

__device__ __forceinline__ uint64_t drain_limit(const CtaCtl* ctl)
{
    return ctl->wait_ns > kWaitTimeoutNs ? ctl->wait_ns : kWaitTimeoutNs;
}

__device__ __forceinline__ void record_timeout(uint32_t where)
{
    if (atomicCAS(&g_status[0], 0u, static_cast<uint32_t>(FA_ERR_DEVICE_TIMEOUT)) == 0u) {
        g_status[1] = where;
        g_status[2] = blockIdx.x;
    }
}

// Single-thread bounded wait.  Returns false (and raises the CTA abort flag) if the
// phase did not complete within ctl->wait_ns, or if another wait already aborted.
// The _inl forms are for kernels that change per-warpgroup register budgets
// (setmaxnreg): their code may not call out-of-line functions.
__device__ __forceinline__ bool wait_bar_inl(uint32_t bar, uint32_t parity, CtaCtl* ctl, uint32_t where)
{
    if (mbar_try_wait(bar, parity)) return true;
    volatile uint32_t* abort = &ctl->abort;
    // the limit is read from shared memory at each check rather than held in registers
    // (code under a tight setmaxnreg budget inlines this loop)
    volatile const uint64_t* limit = &ctl->wait_ns;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > *limit) {
                *abort = 1u;
                record_timeout(where);
                return false;
            }
        }
    }
}

__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, CtaCtl* ctl, uint32_t where)
{
    return wait_bar_inl(bar, parity, ctl, where);
}

// Bounded wait that ignores the abort flag: used while draining in-flight copies or
// MMAs before the CTA exits, which always complete on their own.
__device__ __forceinline__ bool drain_wait_inl(uint32_t bar, uint32_t parity, uint32_t where,
                                               uint64_t limit = kWaitTimeoutNs)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit) {
            record_timeout(where);
            return false;
        }
    }
    return true;
}

__device__ __noinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint32_t where, uint64_t limit)
{
    return drain_wait_inl(bar, parity, where, limit);
}

// The timed waits, inlined (INL) or called.  Code that runs under a setmaxnreg budget
// other than the launch's must not call functions, so it takes the inlined form.
template <bool INL>
__device__ __forceinline__ bool wait_bar_t(uint32_t bar, uint32_t parity, CtaCtl* ctl, uint32_t where)
{
    if constexpr (INL) return wait_bar_inl(bar, parity, ctl, where);
    else return wait_bar(bar, parity, ctl, where);
}
template <bool INL>
__device__ __forceinline__ bool drain_wait_t(uint32_t bar, uint32_t parity, uint32_t where,
                                             uint64_t limit = kWaitTimeoutNs)
{
    if constexpr (INL) return drain_wait_inl(bar, parity, where, limit);
    else return drain_wait(bar, parity, where, limit);
}

// Single-thread wait: one inline probe (SPIN: a bounded non-suspending poll), then the
// timed wait.
template <bool INL = false, bool SPIN = false>
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, CtaCtl* ctl,
                                          uint32_t where)
{
    if constexpr (SPIN) {
        for (uint32_t i = 0; i < kSpinPolls; ++i)
            if (mbar_test_wait(bar, parity)) return true;
    } else {
        if (mbar_try_wait(bar, parity)) return true;
    }
    if constexpr (INL) return wait_bar_inl(bar, parity, ctl, where);
    else return wait_bar(bar, parity, ctl, where);
}

// Warp-wide wait: lane 0 polls (its successful wait is the acquire), the result is
// broadcast, and a warp barrier -- which orders memory among the lanes, unlike the
// shuffle -- makes everything lane 0 acquired visible to the other lanes' later loads.
template <bool INL = false, bool SPIN = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, CtaCtl* ctl,
                                          uint32_t where)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_fast<INL, SPIN>(bar, parity, ctl, where) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// MMA-issue primitives for either a warp-converged issuer (WARP: all 32 lanes call
// them; each tcgen05 op is executed by one elected lane, which keeps descriptors
// warp-uniform) or a single issuing thread.
template <bool WARP, bool INL = false, bool SPIN = false>
struct Issuer {
    __device__ static bool wait(uint32_t bar, uint32_t parity, CtaCtl* ctl, uint32_t where)
    {
        if constexpr (WARP) return warp_wait<INL, SPIN>(bar, parity, ctl, where);
        else return wait_fast<INL, SPIN>(bar, parity, ctl, where);
    }
    __device__ static void ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
    {
        if constexpr (WARP) mma_ss_w(d, a, b, idesc, acc);
        else mma_ss(d, a, b, idesc, acc);
    }
    __device__ static void ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc)
    {
        if constexpr (WARP) mma_ts_w(d, a, b, idesc, acc);
        else mma_ts(d, a, b, idesc, acc);
    }
    __device__ static void commit(uint32_t bar)
    {
        if constexpr (WARP) mma_commit_w(bar);
        else mma_commit(bar);
    }
};

// ---------------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 f32x2 arithmetic on the FMA pipe: two lanes of work per
// instruction).  A pair lives in one 64-bit register, `lo` in the low half.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v)
{
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// exp2_fma on a pair: the range reduction in packed fp32 (x arrives packed), the cubic
// in scalar FMAs with immediate coefficients (no registers held for constants), and
// 2^n applied with one integer multiply-add per value: the bits of t = x + 1.5*2^23
// are 0x4B400000 + n, and (t_bits * 2^23) mod 2^32 = n << 23.
__device__ __forceinline__ uint32_t imad_u32(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ void exp2_fma_x2(uint64_t x2, float& e0, float& e1)
{
    const float2 xc = f2unpack(x2);
    const uint64_t x = f2pack(fmaxf(xc.x, -126.0f), fmaxf(xc.y, -126.0f));
    const uint64_t t = fadd2(x, f2pack(12582912.0f, 12582912.0f));
    const uint64_t n = fadd2(t, f2pack(-12582912.0f, -12582912.0f));
    const float2 f = f2unpack(ffma2(n, f2pack(-1.0f, -1.0f), x));  // x - n, exact
    float p0 = fmaf(FA_EXP2_C3, f.x, FA_EXP2_C2), p1 = fmaf(FA_EXP2_C3, f.y, FA_EXP2_C2);
    p0 = fmaf(p0, f.x, FA_EXP2_C1);
    p1 = fmaf(p1, f.y, FA_EXP2_C1);
    p0 = fmaf(p0, f.x, FA_EXP2_C0);
    p1 = fmaf(p1, f.y, FA_EXP2_C0);
    const float2 tf = f2unpack(t);
    e0 = __uint_as_float(imad_u32(__float_as_uint(tf.x), 1u << 23, __float_as_uint(p0)));
    e1 = __uint_as_float(imad_u32(__float_as_uint(tf.y), 1u << 23, __float_as_uint(p1)));
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

// Packing of P (values in [0, 2^8]) for the P V product: one conversion instruction
// per pair (round to nearest even), measured cheaper than integer rounding and a byte
// permute on sm_100.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2_p(float lo, float hi)
{
    return pack2<BF16>(lo, hi);
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
