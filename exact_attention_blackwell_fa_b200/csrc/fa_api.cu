// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor
// maps, device checks and kernel launches.  Every entry point validates first and
// launches nothing on an invalid argument; there is no alternative code path.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_wide.cuh"
#include "fa_fwd.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 4-D map over a [B, S, H, d] 16-bit tensor; one box = 64 head-dim columns x box_rows
// rows of one (batch, head), 128-byte swizzled.  Rows past S read as zero.
bool make_tmap(CUtensorMap* m, const void* ptr, int B, int S, int H, int d, bool bf16,
               int box_rows = 128, int box_heads = 1)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2,
                                   (cuuint64_t)S * H * d * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
               const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sm_count = 0;
    bool ok = false;  // compute capability 10.0 (B200 class, sm_100a code runs)
};

constexpr int kMaxDevices = 64;

fa_status device_info(DeviceInfo* out)
{
    static DeviceInfo cache[kMaxDevices];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev].sm_count == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        cache[dev].sm_count = sms;
        cache[dev].ok = (major == 10 && minor == 0);
    }
    *out = cache[dev];
    return out->ok ? FA_OK : FA_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int Sq, int Sk, int Hq, int Hkv, int d, float scale, fa_dtype dt)
{
    if (B < 1 || Sq < 1 || Sk < 1 || Hq < 1 || Hkv < 1) return FA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return FA_ERR_INVALID_ARG;
    if (d != 128 && d != 192 && d != 256 && d != 384 && d != 512) return FA_ERR_UNSUPPORTED;
    if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_UNSUPPORTED;
    // element counts must stay inside the 32-bit row indices the kernels use
    const long long rows_q = (long long)B * Sq * Hq, rows_k = (long long)B * Sk * Hkv;
    if (rows_q >= (1LL << 31) || rows_k >= (1LL << 31)) return FA_ERR_INVALID_ARG;
    return FA_OK;
}

int chunk_heads_for(int B, int Hq, int group, int Sk, int d)
{
    // heads whose K and V together stay well inside the 126-MB L2
    const double kv_bytes = 2.0 * Sk * d * 2.0 / group;
    const double budget = 48.0 * 1024 * 1024;
    int c = static_cast<int>(budget / (kv_bytes > 1.0 ? kv_bytes : 1.0));
    if (c < 1) c = 1;
    if (c > B * Hq) c = B * Hq;
    return c;
}

template <typename K>
fa_status set_smem(K kernel, uint32_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes)) == cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
}

// A kernel that moves registers between warpgroups with setmaxnreg assumes the launch
// gives every thread exactly `launch_regs`; a build compiled to another count could
// leave an increase waiting forever, so it is refused before any launch.
template <typename K>
fa_status check_regs(K kernel, int launch_regs)
{
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return FA_ERR_CUDA;
    return a.numRegs == launch_regs ? FA_OK : FA_ERR_UNSUPPORTED;
}

int g_inject = 0;
std::mutex g_inject_mu;
std::atomic<int> g_schedule{FA_SCHED_AUTO};
std::atomic<int> g_exp2_emu{-1};  // -1: the per-head-dim default
std::atomic<uint64_t> g_wait_ns{fa::kWaitTimeoutNs};  // limit of a kernel's pipeline waits

int take_inject()
{
    std::lock_guard<std::mutex> lk(g_inject_mu);
    int v = g_inject;
    g_inject = 0;
    return v;
}

template <bool BF16>
fa_status launch_bwd_d128(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const fa::BwdParams& p, int sm_count,
                          cudaStream_t stream)
{
    using C = fa::BwdCfg<BF16>;
    static const fa_status regs_ok = check_regs(fa::fa_bwd_dkdv_kernel<BF16>, C::REG_LAUNCH);
    if (regs_ok != FA_OK) return regs_ok;
    fa_status st = set_smem(fa::fa_bwd_dkdv_kernel<BF16>, C::SMEM_BYTES);
    if (st != FA_OK) return st;
    const long long pre_rows = (long long)p.B * p.Hq * p.Sq_pad;
    fa::fa_bwd_pre_kernel<128, BF16><<<(unsigned)((pre_rows + 7) / 8), 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    const int grid = p.num_units < sm_count ? p.num_units : sm_count;
    fa::fa_bwd_dkdv_kernel<BF16><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    const long long dq_rows = (long long)p.B * p.Sq * p.Hq;
    fa::fa_bwd_dq_kernel<128, BF16><<<(unsigned)((dq_rows + 7) / 8), 256, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16>
fa_status launch_bwd_wide(const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv64,
                          const CUtensorMap& tdo, const fa::BwdParams& p, int sm_count,
                          cudaStream_t stream)
{
    using C = fa::BwdWideCfg<D, BF16>;
    static const fa_status regs_ok = check_regs(fa::fa_bwd_dkdv_wide_kernel<D, BF16>, C::REG_LAUNCH);
    if (regs_ok != FA_OK) return regs_ok;
    fa_status st = set_smem(fa::fa_bwd_dkdv_wide_kernel<D, BF16>, C::SMEM_BYTES);
    if (st != FA_OK) return st;
    const long long pre_rows = (long long)p.B * p.Hq * p.Sq_pad;
    fa::fa_bwd_pre_kernel<D, BF16><<<(unsigned)((pre_rows + 7) / 8), 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    const int grid = p.num_units < sm_count ? p.num_units : sm_count;
    fa::fa_bwd_dkdv_wide_kernel<D, BF16><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk64, tv64, tdo, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    const long long dq_rows = (long long)p.B * p.Sq * p.Hq;
    fa::fa_bwd_dq_kernel<D, BF16><<<(unsigned)((dq_rows + 7) / 8), 256, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16, int EMU>
fa_status launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     fa::FwdParams p, int sm_count, cudaStream_t stream)
{
    using C = fa::FwdCfg<D, BF16>;
    if constexpr (C::REG_SPLIT) {
        static const fa_status regs_ok = check_regs(fa::fa_fwd_kernel<D, BF16, EMU>, C::REG_LAUNCH);
        if (regs_ok != FA_OK) return regs_ok;
    }
    fa_status st = set_smem(fa::fa_fwd_kernel<D, BF16, EMU>, C::SMEM_BYTES);
    if (st != FA_OK) return st;

    // cluster launch control: one CTA per unit, the running ones take the rest
    const int grid = p.clc ? p.num_tiles : (p.num_tiles < sm_count ? p.num_tiles : sm_count);
    fa::fa_fwd_kernel<D, BF16, EMU><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// query rows per forward work unit: two 128-row Q tiles at head_dim 128, one otherwise
int fwd_unit_rows(int d) { return d == 128 ? 256 : 128; }

// forward work units per Q tile: head dims 384 and 512 split V / O into two halves
int fwd_vparts(int d) { return d > 256 ? 2 : 1; }

// Exponential pairs of every four that the forward computes with the FMA-pipe cubic
// when the caller has not chosen (fa_set_exp2_emulation(-1)), per head dim.
int exp2_emulation_default(int d)
{
    (void)d;
    return 0;
}

template <int D, bool BF16>
fa_status launch_fwd_emu(int emu, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const fa::FwdParams& p, int sm_count, cudaStream_t s)
{
    switch (emu) {
    case 0: return launch_fwd<D, BF16, 0>(tq, tk, tv, p, sm_count, s);
    case 1: return launch_fwd<D, BF16, 1>(tq, tk, tv, p, sm_count, s);
    case 2: return launch_fwd<D, BF16, 2>(tq, tk, tv, p, sm_count, s);
    case 3: return launch_fwd<D, BF16, 3>(tq, tk, tv, p, sm_count, s);
    default: return FA_ERR_INVALID_ARG;
    }
}

fa_status launch_fwd_any(int d, bool bf16, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         fa::FwdParams p, int sm_count, cudaStream_t s)
{
    // dynamic unit order (cluster launch control) when selected, or by default for
    // causal launches over >= 4096 keys, and there are more units than SMs
    const int mode = g_schedule.load(std::memory_order_relaxed);
    const bool dynamic = mode == FA_SCHED_CLC || (mode == FA_SCHED_AUTO && p.causal && p.Sk >= 4096);
    p.clc = (dynamic && p.num_tiles > sm_count) ? 1 : 0;
    int emu = g_exp2_emu.load(std::memory_order_relaxed);
    if (emu < 0) emu = exp2_emulation_default(d);
    switch (d) {
    case 128: return bf16 ? launch_fwd_emu<128, true>(emu, tq, tk, tv, p, sm_count, s)
                          : launch_fwd_emu<128, false>(emu, tq, tk, tv, p, sm_count, s);
    case 192: return bf16 ? launch_fwd_emu<192, true>(emu, tq, tk, tv, p, sm_count, s)
                          : launch_fwd_emu<192, false>(emu, tq, tk, tv, p, sm_count, s);
    case 256: return bf16 ? launch_fwd_emu<256, true>(emu, tq, tk, tv, p, sm_count, s)
                          : launch_fwd_emu<256, false>(emu, tq, tk, tv, p, sm_count, s);
    case 384: return bf16 ? launch_fwd_emu<384, true>(emu, tq, tk, tv, p, sm_count, s)
                          : launch_fwd_emu<384, false>(emu, tq, tk, tv, p, sm_count, s);
    case 512: return bf16 ? launch_fwd_emu<512, true>(emu, tq, tk, tv, p, sm_count, s)
                          : launch_fwd_emu<512, false>(emu, tq, tk, tv, p, sm_count, s);
    default: return FA_ERR_UNSUPPORTED;
    }
}

template <int D>
void launch_combine(bool bf16, const fa::FwdParams& p, unsigned blocks, cudaStream_t s)
{
    if (bf16) fa::fa_fwd_combine_kernel<D, true><<<blocks, 256, 0, s>>>(p);
    else fa::fa_fwd_combine_kernel<D, false><<<blocks, 256, 0, s>>>(p);
}

}  // namespace

namespace fa {
// Test hook kernel: one thread per pair of values, exactly the kernels' exp2 forms.
__global__ void fa_debug_exp2_kernel(const float* x, float* y, int n, int mode)
{
    const int pr = blockIdx.x * blockDim.x + threadIdx.x;
    const int i0 = 2 * pr, i1 = 2 * pr + 1;
    if (i0 >= n) return;
    const float x0 = x[i0], x1 = i1 < n ? x[i1] : x0;
    float e0, e1;
    if (mode == 0) {
        exp2_fma_x2(f2pack(x0, x1), e0, e1);
    } else {
        e0 = ex2_sfu(x0);
        e1 = ex2_sfu(x1);
    }
    y[i0] = e0;
    if (i1 < n) y[i1] = e1;
}
}  // namespace fa

extern "C" {

// Dense forward; splits > 1 runs the split-KV form with partials in `workspace`.
static fa_status fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                            int Sk, int Hq, int Hkv, int d, int causal, float scale, fa_dtype dt, int splits,
                            void* workspace, fa_stream stream)
{
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    fa_status st = check_common(B, Sq, Sk, Hq, Hkv, d, scale, dt);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    DeviceInfo di;
    st = device_info(&di);
    if (st != FA_OK) return st;
    const bool bf16 = dt == FA_BF16;
    // Pack GQA: with few queries per head, the query heads that share a KV head fill the
    // rows of a Q tile together (the group size must divide the 128-row tile)
    const int group = Hq / Hkv;
    const int pack = (group > 1 && group <= 16 && (group & (group - 1)) == 0 && Sq < 256) ? group : 1;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, q, B, Sq, Hq, d, bf16, 128 / pack, pack) || !make_tmap(&tk, k, B, Sk, Hkv, d, bf16) ||
        !make_tmap(&tv, v, B, Sk, Hkv, d, bf16))
        return FA_ERR_CUDA;
    fa::FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.Sq_alloc = Sq;
    p.pack = pack;
    p.splits = splits;
    if (splits > 1) {
        const size_t part_rows = (size_t)splits * B * Hq * Sq;
        p.opart = static_cast<float*>(workspace);
        p.lsepart = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             fa::bwd_round256(part_rows * d * 4));
    }
    p.B = B;
    p.Sq = Sq;
    p.Sk = Sk;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.group = Hq / Hkv;
    const int unit = fwd_unit_rows(d);
    p.num_m = (Sq * pack + unit - 1) / unit;
    p.num_tiles = B * (pack > 1 ? Hkv : Hq) * p.num_m * fwd_vparts(d) * splits;
    p.chunk_heads = pack > 1 ? chunk_heads_for(B, Hkv, 1, Sk, d) : chunk_heads_for(B, Hq, p.group, Sk, d);
    p.causal = causal ? 1 : 0;
    p.inject = take_inject();
    p.sl2 = scale * 1.4426950408889634f;
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = launch_fwd_any(d, bf16, tq, tk, tv, p, di.sm_count, s);
    if (st != FA_OK || splits == 1) return st;
    const long long rows = (long long)B * Hq * Sq;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (d == 128) launch_combine<128>(bf16, p, blocks, s);
    else if (d == 192) launch_combine<192>(bf16, p, blocks, s);
    else if (d == 256) launch_combine<256>(bf16, p, blocks, s);
    else if (d == 384) launch_combine<384>(bf16, p, blocks, s);
    else launch_combine<512>(bf16, p, blocks, s);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                 int Sk, int Hq, int Hkv, int d, int causal, float scale, fa_dtype dt,
                 fa_stream stream)
{
    return fwd_common(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, d, causal, scale, dt, 1, nullptr, stream);
}

// Slices for the split-KV forward: the count that minimises (waves of units over the
// SMs) x (KV tiles per slice + a per-unit fixed cost of about two tiles: pipeline
// fill and drain, epilogue, its share of the combine), from 1 to 64 slices of at
// least two tiles each.  A count that leaves a short last wave costs a whole wave.
static int splitkv_auto(int B, int Sq, int Sk, int Hq, int Hkv, int d, int sm_count)
{
    const int group = Hq / Hkv;
    const int pack = (group > 1 && group <= 16 && (group & (group - 1)) == 0 && Sq < 256) ? group : 1;
    const int unit = fwd_unit_rows(d);
    const long long units =
        (long long)B * (pack > 1 ? Hkv : Hq) * ((Sq * pack + unit - 1) / unit) * fwd_vparts(d);
    const int nk = (Sk + 127) / 128;
    const int smax = nk / 2 < 64 ? nk / 2 : 64;
    int best = 1;
    long long best_cost = -1;
    for (int s = 1; s <= (smax > 1 ? smax : 1); ++s) {
        const long long waves = (units * s + sm_count - 1) / sm_count;
        const long long cost = waves * ((nk + s - 1) / s + 2);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

size_t fa_fwd_splitkv_workspace_size(int B, int Sq, int Sk, int Hq, int Hkv, int d, int num_splits)
{
    if (B < 1 || Sq < 1 || Sk < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv ||
        (d != 128 && d != 192 && d != 256 && d != 384 && d != 512))
        return 0;
    if (num_splits <= 0) {
        DeviceInfo di;
        if (device_info(&di) != FA_OK) return 0;
        num_splits = splitkv_auto(B, Sq, Sk, Hq, Hkv, d, di.sm_count);
    }
    if (num_splits > 64) num_splits = 64;
    const size_t rows = (size_t)num_splits * B * Hq * Sq;
    return fa::bwd_round256(rows * d * 4) + fa::bwd_round256(rows * 4);
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                         int Sk, int Hq, int Hkv, int d, int causal, float scale, fa_dtype dt, int num_splits,
                         void* workspace, size_t workspace_bytes, fa_stream stream)
{
    if (num_splits > 64) return FA_ERR_INVALID_ARG;
    if (num_splits <= 0) {
        fa_status st = check_common(B, Sq, Sk, Hq, Hkv, d, scale, dt);
        if (st != FA_OK) return st;
        DeviceInfo di;
        st = device_info(&di);
        if (st != FA_OK) return st;
        num_splits = splitkv_auto(B, Sq, Sk, Hq, Hkv, d, di.sm_count);
    }
    if (num_splits > 1) {
        if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_INVALID_ARG;
        if (workspace_bytes < fa_fwd_splitkv_workspace_size(B, Sq, Sk, Hq, Hkv, d, num_splits))
            return FA_ERR_INVALID_ARG;
    }
    return fwd_common(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, d, causal, scale, dt, num_splits, workspace, stream);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, const int* seqused_k, int B,
                        int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv,
                        int d, int causal, float scale, fa_dtype dt, fa_stream stream)
{
    if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
    if (total_q < 1 || total_k < 1) return FA_ERR_INVALID_ARG;
    fa_status st = check_common(B, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, dt);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) | reinterpret_cast<uintptr_t>(cu_seqlens_k) |
         reinterpret_cast<uintptr_t>(seqused_k)) & 3u)
        return FA_ERR_INVALID_ARG;
    DeviceInfo di;
    st = device_info(&di);
    if (st != FA_OK) return st;
    const bool bf16 = dt == FA_BF16;
    // packed tensors: one batch entry of total rows
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, q, 1, total_q, Hq, d, bf16) || !make_tmap(&tk, k, 1, total_k, Hkv, d, bf16) ||
        !make_tmap(&tv, v, 1, total_k, Hkv, d, bf16))
        return FA_ERR_CUDA;
    fa::FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k;
    p.used_k = seqused_k;
    p.Sq_alloc = total_q;
    p.pack = 1;
    p.splits = 1;
    p.B = B;
    p.Sq = max_seqlen_q;
    p.Sk = max_seqlen_k;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.group = Hq / Hkv;
    const int unit = fwd_unit_rows(d);
    p.num_m = (max_seqlen_q + unit - 1) / unit;
    p.num_tiles = B * Hq * p.num_m * fwd_vparts(d);
    p.chunk_heads = chunk_heads_for(B, Hq, p.group, max_seqlen_k, d);
    p.causal = causal ? 1 : 0;
    p.inject = take_inject();
    p.sl2 = scale * 1.4426950408889634f;
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    return launch_fwd_any(d, bf16, tq, tk, tv, p, di.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int Sq, int Hq, int d)
{
    if (B < 1 || Sq < 1 || Hq < 1 || d < 1) return 0;
    return fa::bwd_workspace_bytes(B, Sq, Hq, d);
}

// The backward for B batch entries of (at most) Sq queries and Sk keys; the q-side
// tensors hold Sq_alloc rows per entry and the k-side Sk_alloc (packed sequences:
// one entry of total rows, with cu_q / cu_k / used_k describing the sequences).
static fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, const int* cu_q, const int* cu_k,
                            const int* used_k, int B, int Sq, int Sk, int Sq_alloc, int Sk_alloc, int TB,
                            int Hq, int Hkv, int d, int causal, float scale, fa_dtype dt, void* workspace,
                            size_t workspace_bytes, fa_stream stream)
{
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
        return FA_ERR_INVALID_ARG;
    fa_status st = check_common(B, Sq, Sk, Hq, Hkv, d, scale, dt);
    if (st != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return FA_ERR_INVALID_ARG;
    if (workspace_bytes < fa::bwd_workspace_bytes(B, Sq, Hq, d)) return FA_ERR_INVALID_ARG;
    DeviceInfo di;
    st = device_info(&di);
    if (st != FA_OK) return st;
    const bool bf16 = dt == FA_BF16;
    const int kv_rows = d == 128 ? 128 : 64;  // keys per backward work unit
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tmap(&tq, q, TB, Sq_alloc, Hq, d, bf16) || !make_tmap(&tk, k, TB, Sk_alloc, Hkv, d, bf16, kv_rows) ||
        !make_tmap(&tv, v, TB, Sk_alloc, Hkv, d, bf16, kv_rows) || !make_tmap(&tdo, dout, TB, Sq_alloc, Hq, d, bf16))
        return FA_ERR_CUDA;
    fa::BwdParams p{};
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    const size_t sq_pad = fa::bwd_sq_pad(Sq);
    const size_t rows = (size_t)B * Hq * sq_pad;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.Dv = reinterpret_cast<float*>(ws);
    p.L2 = reinterpret_cast<float*>(ws + fa::bwd_round256(rows * 4));
    p.dqacc = reinterpret_cast<float*>(ws + 2 * fa::bwd_round256(rows * 4));
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.used_k = used_k;
    p.Sq_alloc = Sq_alloc;
    p.Sk_alloc = Sk_alloc;
    p.B = B;
    p.Sq = Sq;
    p.Sk = Sk;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.group = Hq / Hkv;
    p.Sq_pad = (int)sq_pad;
    p.num_n = (Sk + kv_rows - 1) / kv_rows;
    p.num_m = (Sq + 127) / 128;
    // head dims 384 / 512: each key block is two units, one per half of the output dims
    p.num_units = B * Hkv * p.num_n * (d > 256 ? 2 : 1);
    // KV heads whose Q and dO streams stay inside L2 together
    {
        const double qdo_bytes = 2.0 * Sq * d * 2.0 * p.group;
        int c = (int)(48.0 * 1024 * 1024 / (qdo_bytes > 1.0 ? qdo_bytes : 1.0));
        if (c < 1) c = 1;
        if (c > B * Hkv) c = B * Hkv;
        p.chunk_heads = c;
    }
    p.causal = causal ? 1 : 0;
    p.scale = scale;
    p.sl2 = scale * 1.4426950408889634f;
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 512)
        return bf16 ? launch_bwd_wide<512, true>(tq, tk, tv, tdo, p, di.sm_count, s)
                    : launch_bwd_wide<512, false>(tq, tk, tv, tdo, p, di.sm_count, s);
    if (d == 384)
        return bf16 ? launch_bwd_wide<384, true>(tq, tk, tv, tdo, p, di.sm_count, s)
                    : launch_bwd_wide<384, false>(tq, tk, tv, tdo, p, di.sm_count, s);
    if (d == 256)
        return bf16 ? launch_bwd_wide<256, true>(tq, tk, tv, tdo, p, di.sm_count, s)
                    : launch_bwd_wide<256, false>(tq, tk, tv, tdo, p, di.sm_count, s);
    if (d == 192)
        return bf16 ? launch_bwd_wide<192, true>(tq, tk, tv, tdo, p, di.sm_count, s)
                    : launch_bwd_wide<192, false>(tq, tk, tv, tdo, p, di.sm_count, s);
    return bf16 ? launch_bwd_d128<true>(tq, tk, tv, tdo, p, di.sm_count, s)
                : launch_bwd_d128<false>(tq, tk, tv, tdo, p, di.sm_count, s);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq,
                 int Hkv, int d, int causal, float scale, fa_dtype dt, void* workspace,
                 size_t workspace_bytes, fa_stream stream)
{
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, nullptr, nullptr, nullptr, B, Sq, Sk, Sq, Sk, B, Hq, Hkv, d,
                      causal, scale, dt, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, const int* seqused_k, int B, int max_seqlen_q,
                        int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, int causal,
                        float scale, fa_dtype dt, void* workspace, size_t workspace_bytes, fa_stream stream)
{
    if (!cu_seqlens_q || !cu_seqlens_k || total_q < 1 || total_k < 1) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) | reinterpret_cast<uintptr_t>(cu_seqlens_k) |
         reinterpret_cast<uintptr_t>(seqused_k)) & 3u)
        return FA_ERR_INVALID_ARG;
    return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, seqused_k, B, max_seqlen_q,
                      max_seqlen_k, total_q, total_k, 1, Hq, Hkv, d, causal, scale, dt, workspace, workspace_bytes,
                      stream);
}

const char* fa_status_string(fa_status s)
{
    switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid size, pointer, alignment or scale";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head_dim, dtype or GPU not supported";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    case FA_ERR_SCRATCH_LIMIT:
        return "FA_ERR_SCRATCH_LIMIT: problem needs more scratch than fa_bwd_noalloc's built-in array";
    }
    return "unknown fa_status";
}

fa_status fa_last_device_status(fa_stream stream, uint32_t* detail)
{
    uint32_t h[4] = {0, 0, 0, 0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyFromSymbolAsync(h, fa::g_status, sizeof(h), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return FA_ERR_CUDA;
    if (detail) *detail = h[1];
    return static_cast<fa_status>(h[0]);
}

fa_status fa_clear_device_status(fa_stream stream)
{
    static const uint32_t zero[4] = {0, 0, 0, 0};
    return cudaMemcpyToSymbolAsync(fa::g_status, zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
}

fa_status fa_debug_exp2(const float* x, float* y, int n, int mode, fa_stream stream)
{
    if (n < 0 || (mode != 0 && mode != 1) || (n > 0 && (x == nullptr || y == nullptr))) return FA_ERR_INVALID_ARG;
    if (n == 0) return FA_OK;
    const int pairs = (n + 1) / 2;
    const int threads = 256;
    const int blocks = (pairs + threads - 1) / threads;
    fa::fa_debug_exp2_kernel<<<blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_set_unit_schedule(int mode)
{
    if (mode != FA_SCHED_STATIC && mode != FA_SCHED_CLC && mode != FA_SCHED_AUTO) return FA_ERR_INVALID_ARG;
    g_schedule.store(mode, std::memory_order_relaxed);
    return FA_OK;
}

fa_status fa_set_exp2_emulation(int pairs_of_4)
{
    if (pairs_of_4 < -1 || pairs_of_4 > 3) return FA_ERR_INVALID_ARG;
    g_exp2_emu.store(pairs_of_4, std::memory_order_relaxed);
    return FA_OK;
}

fa_status fa_set_wait_timeout_ms(int ms)
{
    if (ms < 1 || ms > 600000) return FA_ERR_INVALID_ARG;
    g_wait_ns.store(static_cast<uint64_t>(ms) * 1000000ull, std::memory_order_relaxed);
    return FA_OK;
}

fa_status fa_debug_inject(int mode)
{
    if (mode != 0 && mode != 1) return FA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_inject_mu);
    g_inject = mode;
    return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// fa_bwd_noalloc: fa_bwd with its scratch in a fixed device array, for callers that
// cannot allocate device memory (a caller-owned pool or arena that forbids
// cudaMalloc, loops that cannot afford the synchronisation cudaMalloc/cudaFree imply,
// an embedded host without a device allocator of its own).  Every call on a device
// shares the array; calls whose kernels overlap on the GPU race on it.
// ---------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_noalloc_scratch, looked up once per device.  In host code the
// array's name is only a host-side stand-in, so kernels must be given this address.
fa_status noalloc_scratch(void** out)
{
    static void* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return FA_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk,
                                    void* dv, int B, int Sq, int Sk, int Hq, int Hkv, int d,
                                    int causal, float scale, fa_dtype dt, fa_stream stream)
{
    fa_status st = check_common(B, Sq, Sk, Hq, Hkv, d, scale, dt);
    if (st != FA_OK) return st;
    if (fa::bwd_workspace_bytes(B, Sq, Hq, d) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != FA_OK) return st;
    return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Sq, Sk, Hq, Hkv, d, causal, scale, dt,
                  scratch, FA_NOALLOC_SCRATCH_BYTES, stream);
}
