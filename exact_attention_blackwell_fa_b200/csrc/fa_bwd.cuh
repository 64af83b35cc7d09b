// fa_bwd.cuh -- exact attention backward for sm_100a.
//
// Given Q, K, V, O, LSE and dO, computes dQ, dK, dV of O = softmax(scale Q K^T) V
// (the backward is listed as merged for SM100 in "[RFC] FA4 -- head_dim=256 &
// head_dim=512", Phase 1 table; the arithmetic is the chain rule of the forward):
//
//   P_ij  = exp(scale q_i.k_j - LSE_i)          (recomputed, never stored in HBM)
//   dP_ij = dO_i . v_j,   D_i = dO_i . O_i,   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
//
// Three kernels on one stream:
//   1. preprocess: D_i = rowsum(dO * O), LSE in log2 units, zero the fp32 dQ
//      accumulator (rows padded to a multiple of 128);
//   2. dK/dV kernel, persistent, one work unit = one block of 128 key rows of one
//      (batch, KV head); it loops over every query head of the KV group and every
//      block of 128 query rows.  Per step, all in TMEM:
//        S^T = K Q^T,  dP^T = V dO^T            (tcgen05, A and B K-major)
//        two compute warpgroups (thread = key row; one warpgroup per half of the
//        128 query columns): P^T -> TMEM as 16-bit pairs, dS^T -> shared memory
//        dV += P^T dO   (A from TMEM)           dK += dS^T Q   (A K-major)
//        dQ^T = K^T dS^T (both read MN-major; head dims land on the TMEM lanes)
//        -> fp32 reductions into the dQ accumulator by a second warpgroup, one
//        128-byte accumulator segment per warp instruction;
//   3. convert: dQ = scale * accumulator, in the input dtype and layout.
#pragma once

#include <type_traits>
#include <utility>

#include "fa_common.cuh"

namespace fa {

inline size_t bwd_round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline size_t bwd_sq_pad(int Sq) { return (static_cast<size_t>(Sq) + 127) / 128 * 128; }

// workspace = D [B*Hq*Sq_pad] fp32 | LSE*log2(e) [B*Hq*Sq_pad] fp32 | dQacc [.. x d] fp32
inline size_t bwd_workspace_bytes(int B, int Sq, int Hq, int d)
{
    const size_t rows = static_cast<size_t>(B) * Hq * bwd_sq_pad(Sq);
    return 2 * bwd_round256(rows * 4) + bwd_round256(rows * d * 4);
}

struct BwdParams {
    const void* o;
    const void* dout;
    const float* lse;
    float* Dv;     // D_i, padded rows 0
    float* L2;     // LSE_i * log2(e); +inf for padded rows and rows without keys
    float* dqacc;  // [B, Hq, Sq_pad, d] fp32
    void* dq;
    void* dk;
    void* dv;
    // Packed variable-length batches (null for the dense layout): sequence b's
    // queries are rows cu_q[b] .. of the [total_q, Hq, d] tensors, its keys rows
    // cu_k[b] .. of [total_k, Hkv, d], the first used_k[b] of them taking part.
    // Sq / Sk are then the maximum lengths; the workspace stays dense per sequence.
    const int* cu_q;
    const int* cu_k;
    const int* used_k;
    int Sq_alloc, Sk_alloc;  // rows per batch entry of the q- / k-side tensors
    int B, Sq, Sk, Hq, Hkv, group, Sq_pad;
    int num_n;        // key blocks per KV head
    int num_m;        // query blocks per query head
    int num_units;    // B * Hkv * num_n
    int chunk_heads;  // KV heads per L2 group in the unit order
    int causal;
    float scale, sl2;
    uint64_t wait_ns;  // limit of a pipeline wait (see CtaCtl)
};

enum : uint32_t {
    W_BWD_KV_FULL = 0x201, W_BWD_KV_EMPTY, W_BWD_Q_FULL, W_BWD_Q_EMPTY, W_BWD_DO_FULL,
    W_BWD_DO_EMPTY, W_BWD_S_FULL, W_BWD_DP_FULL, W_BWD_P_FULL, W_BWD_DS_FULL, W_BWD_DS_EMPTY,
    W_BWD_DQ_FULL, W_BWD_DQ_EMPTY, W_BWD_DKV_FINAL, W_BWD_DRAIN, W_BWD_SMEM_ALIGN
};

// Rows of batch entry b: the TMA batch coordinate, the tensor rows of its first
// query and key, and its query / key counts.
struct BwdSeq {
    int tb, q_base, k_base, Sq, Sk;
};

__device__ __forceinline__ BwdSeq bwd_seq(const BwdParams& p, int b)
{
    BwdSeq s;
    if (p.cu_q != nullptr) {
        s.tb = 0;
        s.q_base = p.cu_q[b];
        s.k_base = p.cu_k[b];
        const int sq = p.cu_q[b + 1] - s.q_base;
        const int sk = p.used_k != nullptr ? p.used_k[b] : p.cu_k[b + 1] - s.k_base;
        s.Sq = max(0, min(sq, p.Sq));
        s.Sk = max(0, min(sk, p.Sk));
    } else {
        s.tb = b;
        s.q_base = 0;
        s.k_base = 0;
        s.Sq = p.Sq;
        s.Sk = p.Sk;
    }
    return s;
}

// ---------------------------------------------------------------------------------
// 1. preprocess: one warp per padded query row (b, h, i)
// ---------------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p)
{
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const long long total = static_cast<long long>(p.B) * p.Hq * p.Sq_pad;
    if (row >= total) return;
    const int bh = static_cast<int>(row / p.Sq_pad);
    const int i = static_cast<int>(row - static_cast<long long>(bh) * p.Sq_pad);
    const int b = bh / p.Hq, h = bh - b * p.Hq;
    const BwdSeq sq = bwd_seq(p, b);
    const size_t trow = static_cast<size_t>(sq.tb) * p.Sq_alloc + sq.q_base + i;  // tensor row
    float acc = 0.0f;
    if (i < sq.Sq) {
        const size_t off = (trow * p.Hq + h) * D + lane * (D / 32);
        constexpr int NW = D / 64;  // 32-bit words per lane (two 16-bit values each)
        uint32_t ow[NW], dw[NW];
        const uint16_t* o16 = static_cast<const uint16_t*>(p.o) + off;
        const uint16_t* d16 = static_cast<const uint16_t*>(p.dout) + off;
        if constexpr (NW == 3) {  // 12 bytes per lane: 4-byte aligned only
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                ow[w] = reinterpret_cast<const uint32_t*>(o16)[w];
                dw[w] = reinterpret_cast<const uint32_t*>(d16)[w];
            }
        } else if constexpr (NW % 4 != 0) {  // 8 or 24 bytes per lane: 8-byte aligned
#pragma unroll
            for (int w = 0; w < NW; w += 2) {
                const uint2 a = reinterpret_cast<const uint2*>(o16)[w / 2];
                const uint2 c = reinterpret_cast<const uint2*>(d16)[w / 2];
                ow[w] = a.x; ow[w + 1] = a.y; dw[w] = c.x; dw[w + 1] = c.y;
            }
        } else {  // 16 or 32 bytes per lane
#pragma unroll
            for (int w = 0; w < NW; w += 4) {
                const uint4 a = reinterpret_cast<const uint4*>(o16)[w / 4];
                const uint4 c = reinterpret_cast<const uint4*>(d16)[w / 4];
                ow[w] = a.x; ow[w + 1] = a.y; ow[w + 2] = a.z; ow[w + 3] = a.w;
                dw[w] = c.x; dw[w + 1] = c.y; dw[w + 2] = c.z; dw[w + 3] = c.w;
            }
        }
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float2 x = unpack2<BF16>(ow[w]);
            const float2 y = unpack2<BF16>(dw[w]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) {
        p.Dv[row] = acc;
        float l2 = INFINITY;
        if (i < sq.Sq) {
            const float lse = p.lse[(static_cast<size_t>(sq.tb) * p.Hq + h) * p.Sq_alloc + sq.q_base + i];
            if (lse != -INFINITY) l2 = lse * 1.4426950408889634f;
        }
        p.L2[row] = l2;
    }
    float4* z = reinterpret_cast<float4*>(p.dqacc + static_cast<size_t>(row) * D);
#pragma unroll
    for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------------
// 3. convert: one warp per dQ row (b, i, h)
// ---------------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p)
{
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const long long total = static_cast<long long>(p.B) * p.Sq * p.Hq;
    if (row >= total) return;
    const int h = static_cast<int>(row % p.Hq);
    const long long bi = row / p.Hq;
    const int i = static_cast<int>(bi % p.Sq);
    const int b = static_cast<int>(bi / p.Sq);
    const BwdSeq sq = bwd_seq(p, b);
    if (i >= sq.Sq) return;
    const size_t trow = static_cast<size_t>(sq.tb) * p.Sq_alloc + sq.q_base + i;
    const float* src = p.dqacc + ((static_cast<size_t>(b) * p.Hq + h) * p.Sq_pad + i) * D + lane * (D / 32);
    uint16_t* dst = static_cast<uint16_t*>(p.dq) + (trow * p.Hq + h) * D + lane * (D / 32);
    if constexpr (D == 192) {  // 6 values per lane: 8-byte loads, 4-byte stores
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const float2 a = reinterpret_cast<const float2*>(src)[c];
            reinterpret_cast<uint32_t*>(dst)[c] = pack2<BF16>(a.x * p.scale, a.y * p.scale);
        }
    } else if constexpr (D > 256) {  // 12 or 16 values per lane: 16-byte loads, 8-byte stores
#pragma unroll
        for (int c = 0; c < D / 128; ++c) {
            const float4 a = reinterpret_cast<const float4*>(src)[c];
            reinterpret_cast<uint2*>(dst)[c] =
                make_uint2(pack2<BF16>(a.x * p.scale, a.y * p.scale), pack2<BF16>(a.z * p.scale, a.w * p.scale));
        }
    } else if constexpr (D == 128) {
        const float4 a = *reinterpret_cast<const float4*>(src);
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pack2<BF16>(a.x * p.scale, a.y * p.scale), pack2<BF16>(a.z * p.scale, a.w * p.scale));
    } else {
        const float4 a = reinterpret_cast<const float4*>(src)[0];
        const float4 c = reinterpret_cast<const float4*>(src)[1];
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack2<BF16>(a.x * p.scale, a.y * p.scale), pack2<BF16>(a.z * p.scale, a.w * p.scale),
                       pack2<BF16>(c.x * p.scale, c.y * p.scale), pack2<BF16>(c.z * p.scale, c.w * p.scale));
    }
}

// ---------------------------------------------------------------------------------
// 2. dK / dV kernel (head_dim 128)
// ---------------------------------------------------------------------------------
template <bool BF16>
struct BwdCfg {
    static constexpr int D = 128;
    // warps 0-7: compute (two warpgroups, one per 64-query half), 8-11: dQ, 12: MMA,
    // 13: TMA, 14-15: idle (they complete the fourth warpgroup for setmaxnreg)
    static constexpr int THREADS = 512;
    static constexpr int DQ_WARP = 8, MMA_WARP = 12, LOAD_WARP = 13;
    // registers per thread: launched at 128; the MMA/TMA warpgroup gives 16 of them to
    // the dQ warpgroup, which then holds a whole 128-column dQ^T row in registers
    static constexpr uint32_t REG_LAUNCH = 128, REG_DQ = 144, REG_CTRL = 112;
    static_assert(8 * 32 * REG_LAUNCH + 4 * 32 * REG_DQ + 4 * 32 * REG_CTRL <= THREADS * REG_LAUNCH,
                  "register split exceeds the launch budget");
    // lane 0 of the MMA warp issues alone (the converged, elected-lane form measured
    // slower here)
    static constexpr bool WARP_ISSUE = false;
    static constexpr uint32_t TILE = 32768;  // 128 rows x 128 columns x 2 bytes
    // per query block: LSE*log2(e) and D for its 128 rows, staged with the Q tile
    static constexpr uint32_t ROWS_BYTES = 1024;
    static constexpr uint32_t OFF_K = 0, OFF_V = TILE, OFF_Q = 2 * TILE, OFF_DO = 4 * TILE,
                              OFF_DS = 6 * TILE, OFF_ROWS = 7 * TILE,
                              OFF_BAR = OFF_ROWS + 2 * ROWS_BYTES;
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 1, B_Q_FULL = 2, B_Q_EMPTY = 4, B_DO_FULL = 6,
                         B_DO_EMPTY = 8, B_S_FULL = 10, B_DP_FULL = 11, B_P_FULL = 12, B_DS_FULL = 13,
                         B_DS_EMPTY = 14, B_DQ_FULL = 15, B_DQ_EMPTY = 16, B_DKV_FINAL = 17,
                         B_DRAIN = 18, NBAR = 19;
    static constexpr uint32_t OFF_CTL = OFF_BAR + 8 * NBAR;
    // no alignment slack: the dynamic shared memory base must be 1024-byte aligned,
    // which the kernel checks before it touches anything
    static constexpr uint32_t SMEM_BYTES = OFF_CTL + sizeof(CtaCtl);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // TMEM columns
    static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;
    static constexpr uint32_t IDESC_KK = idesc_f16(BF16, 128, 128, false, false);  // S^T, dP^T
    static constexpr uint32_t IDESC_KM = idesc_f16(BF16, 128, 128, false, true);   // dV, dK
    static constexpr uint32_t IDESC_MM = idesc_f16(BF16, 128, 128, true, true);    // dQ
};

struct BwdUnit {
    int b, hkv, n, m_start, nm, T;
    int tb, q_base, k_base, Sq, Sk;  // the batch entry's rows (see BwdSeq)
    bool keys;                       // the unit's key block holds keys of its sequence
};

__device__ __forceinline__ BwdUnit bwd_decode(const BwdParams& p, int t)
{
    const int BH = p.B * p.Hkv;
    const int per_chunk = p.chunk_heads * p.num_n;
    const int c = t / per_chunk;
    const int r = t - c * per_chunk;
    const int first = c * p.chunk_heads;
    const int csize = min(p.chunk_heads, BH - first);
    const int nb = r / csize;  // causal: ascending n = most query blocks first
    const int bh = first + (r - nb * csize);
    BwdUnit u;
    u.b = bh / p.Hkv;
    u.hkv = bh - u.b * p.Hkv;
    u.n = nb;
    const BwdSeq sq = bwd_seq(p, u.b);
    u.tb = sq.tb;
    u.q_base = sq.q_base;
    u.k_base = sq.k_base;
    u.Sq = sq.Sq;
    u.Sk = sq.Sk;
    u.keys = u.n * 128 < u.Sk;
    const int num_m = (u.Sq + 127) / 128;
    int ms = 0;
    if (p.causal) {
        const long long imin = static_cast<long long>(u.n) * 128 - (u.Sk - u.Sq);
        ms = imin <= 0 ? 0 : static_cast<int>(imin / 128);
        if (ms > num_m) ms = num_m;
    }
    u.m_start = ms;
    u.nm = u.keys ? num_m - ms : 0;
    u.T = p.group * u.nm;
    return u;
}

// query head and query block of step s of a unit
__device__ __forceinline__ void bwd_step(const BwdParams& p, const BwdUnit& u, int s, int& h, int& m)
{
    const int hh = s / u.nm;
    m = u.m_start + (s - hh * u.nm);
    h = u.hkv * p.group + hh;
}

// ---- compute warpgroup: P^T and dS^T, then the dK / dV epilogue --------------------
template <bool BF16>
__device__ void bwd_compute(const BwdParams& p, uint32_t tmem, uint32_t sDS, uint32_t sRows,
                            uint32_t bars, CtaCtl* ctl, int wq, int half)
{
    using C = BwdCfg<BF16>;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const int lane = threadIdx.x & 31;
    const int t = wq * 32 + lane;  // key row within the block (= TMEM lane)
    const int q0 = half * 64;      // this warpgroup's query columns: q0 .. q0 + 63
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    // S^T / dP^T columns of this half; P^T goes to the first 32 columns of the half
    // (16-bit pairs), below the S^T columns still to be read
    const uint32_t tS = tmem + lane_off + C::T_S + q0, tDP = tmem + lane_off + C::T_DP + q0;
    auto bar = [&](int i) { return bars + 8u * i; };
    const uint64_t sl2x2 = f2pack(p.sl2, p.sl2);
    uint32_t it = 0, unit_it = 0;
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        const BwdUnit u = bwd_decode(p, ui);
        if (!u.keys) continue;  // past the end of its sequence's keys
        const int j = u.n * 128 + t;  // key row
        // offset of key row j's dK / dV row
        auto grad_off = [&]() {
            return ((static_cast<size_t>(u.tb) * p.Sk_alloc + u.k_base + j) * p.Hkv + u.hkv) * C::D;
        };
        if (u.T == 0) {  // keys that no query of the sequence sees: zero gradients
            if (j < u.Sk) {
                T* const dvrow = static_cast<T*>(p.dv) + grad_off();
                T* const dkrow = static_cast<T*>(p.dk) + grad_off();
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                for (int c = 2 * half; c < 2 * half + 2; ++c)
                    for (int x = 0; x < 4; ++x) {
                        reinterpret_cast<uint4*>(dvrow + c * 32)[x] = z;
                        reinterpret_cast<uint4*>(dkrow + c * 32)[x] = z;
                    }
            }
            continue;
        }
        for (int s = 0; s < u.T; ++s, ++it) {
            int h, m;
            bwd_step(p, u, s, h, m);
            const uint32_t rows = sRows + (it & 1) * C::ROWS_BYTES;  // L2[128] then D[128]
            // key j is visible to query i iff j <= i + (Sk - Sq) (causal) and j < Sk: the
            // key block's rows past the sequence's keys (zeros, or the next sequence's
            // rows of a packed batch) get P = 0
            const bool masked = (p.causal && (u.n * 128 + 127 > m * 128 + u.Sk - u.Sq)) || (u.n * 128 + 128 > u.Sk);
            int jlim = p.causal ? j - (u.Sk - u.Sq) - m * 128 - q0 : -(1 << 30);  // visible iff column c >= jlim
            if (j >= u.Sk) jlim = 1 << 30;
            // the Q-tile barrier also covers the staged row terms
            if (!warp_wait<true, true>(bar(C::B_Q_FULL + (it & 1)), (it >> 1) & 1u, ctl, W_BWD_Q_FULL)) return;
            if (!warp_wait<true, true>(bar(C::B_S_FULL), it & 1u, ctl, W_BWD_S_FULL)) return;
            tc_fence_after();
            // P^T = 2^(S^T scale log2e - LSE log2e), 32 query columns at a time.  The
            // 16-bit P^T words stay in registers for dS: the MMA issues the next S^T into
            // these TMEM columns as soon as dV has consumed them.
            uint32_t ppk[32];
            uint32_t rbuf[2][32];
            tmem_ld32_nowait(tS, rbuf[0]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t (&r)[32] = rbuf[cc & 1];
                tmem_wait_ld_dep(r);
                if (cc + 1 < 2) tmem_ld32_nowait(tS + (cc + 1) * 32, rbuf[(cc + 1) & 1]);
                uint32_t (&pk)[16] = *reinterpret_cast<uint32_t(*)[16]>(&ppk[cc * 16]);
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    float4 l4;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(l4.x), "=f"(l4.y), "=f"(l4.z), "=f"(l4.w)
                                 : "r"(rows + (q0 + cc * 32 + k4 * 4) * 4u));
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        const int k = k4 * 4 + e;
                        const float la = e == 0 ? l4.x : l4.z, lb = e == 0 ? l4.y : l4.w;
                        const float2 x = f2unpack(ffma2(f2pack(__uint_as_float(r[k]), __uint_as_float(r[k + 1])),
                                                        sl2x2, f2pack(-la, -lb)));
                        // all on the SFU: 128x128 exponentials per step are ~1k SFU cycles,
                        // well under the step's tensor time, and this warpgroup has no
                        // spare warps to hide the longer FMA-pipe sequence
                        float e0 = ex2_sfu(x.x), e1 = ex2_sfu(x.y);
                        if (masked) {
                            const int c = cc * 32 + k;
                            if (c < jlim) e0 = 0.0f;
                            if (c + 1 < jlim) e1 = 0.0f;
                        }
                        pk[k >> 1] = pack2<BF16>(e0, e1);
                    }
                }
                tmem_st16(tS + cc * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL));

            // dS^T = P^T (dP^T - D), 32 query columns at a time (next chunk's load in flight)
            if (!warp_wait<true, true>(bar(C::B_DP_FULL), it & 1u, ctl, W_BWD_DP_FULL)) return;
            if (!warp_wait<true, true>(bar(C::B_DS_EMPTY), (it & 1u) ^ 1u, ctl, W_BWD_DS_EMPTY)) return;
            tc_fence_after();
            tmem_ld32_nowait(tDP, rbuf[0]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t (&r)[32] = rbuf[cc & 1];
                tmem_wait_ld_dep(r);
                if (cc + 1 < 2) tmem_ld32_nowait(tDP + (cc + 1) * 32, rbuf[(cc + 1) & 1]);
#pragma unroll
                for (int g = 0; g < 4; ++g) {  // 8 query columns -> one 16-byte chunk
                    float4 da, db;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(da.x), "=f"(da.y), "=f"(da.z), "=f"(da.w)
                                 : "r"(rows + 512u + (q0 + cc * 32 + g * 8) * 4u));
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(db.x), "=f"(db.y), "=f"(db.z), "=f"(db.w)
                                 : "r"(rows + 512u + (q0 + cc * 32 + g * 8 + 4) * 4u));
                    const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
                    uint32_t q4[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int k = g * 8 + w * 2;  // column within the chunk
                        const float2 pp = unpack2<BF16>(ppk[cc * 16 + (k >> 1)]);
                        q4[w] = pack2<BF16>(pp.x * (__uint_as_float(r[k]) - dv[w * 2]),
                                            pp.y * (__uint_as_float(r[k + 1]) - dv[w * 2 + 1]));
                    }
                    const int col8 = half * 8 + cc * 4 + g;  // 8-column group 0..15
                    const uint32_t addr = sDS + (col8 >> 3) * 16384u + t * 128u +
                                          ((static_cast<uint32_t>(col8 & 7) ^ (t & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(q4[0]),
                                 "r"(q4[1]), "r"(q4[2]), "r"(q4[3])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DS_FULL));
        }
        // epilogue: dV and dK rows of this key block
        if (!warp_wait<true, true>(bar(C::B_DKV_FINAL), unit_it & 1u, ctl, W_BWD_DKV_FINAL)) return;
        ++unit_it;
        tc_fence_after();
        const bool row_ok = j < u.Sk;
        T* const dvrow = static_cast<T*>(p.dv) + grad_off();
        T* const dkrow = static_cast<T*>(p.dk) + grad_off();
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const float mul = which == 0 ? 1.0f : p.scale;
            T* dst = which == 0 ? dvrow : dkrow;
            const uint32_t col = which == 0 ? C::T_DV : C::T_DK;
#pragma unroll 1
            for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
                uint32_t r[32];
                tmem_ld32_wait(tmem + lane_off + col + cc * 32, r);
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    pk[k] = pack2<BF16>(__uint_as_float(r[2 * k]) * mul, __uint_as_float(r[2 * k + 1]) * mul);
                if (row_ok) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
                    d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    d4[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
                    d4[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
                }
            }
        }
        tc_fence_before();
    }
}

// dst[i * STRIDE bytes] += r[i] for every i, from one base address with immediate
// offsets (no per-row address registers)
template <int OFF>
__device__ __forceinline__ void red_at(float* dst, uint32_t v)
{
    asm volatile("red.global.add.f32 [%0+%2], %1;" ::"l"(dst), "f"(__uint_as_float(v)), "n"(OFF) : "memory");
}
template <int STRIDE, size_t... I>
__device__ __forceinline__ void red_rows(float* dst, const uint32_t (&r)[sizeof...(I)], std::index_sequence<I...>)
{
    (red_at<static_cast<int>(I) * STRIDE>(dst, r[I]), ...);
}

// ---- dQ warpgroup: TMEM -> registers -> fp32 vector reductions ----------------------
template <bool BF16>
__device__ void bwd_dq_reduce(const BwdParams& p, uint32_t tmem, uint32_t bars, CtaCtl* ctl, int wq)
{
    using C = BwdCfg<BF16>;
    const int lane = threadIdx.x & 31;
    const int t = wq * 32 + lane;  // head dim (= TMEM lane of dQ^T)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    auto bar = [&](int i) { return bars + 8u * i; };
    uint32_t it = 0;
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        const BwdUnit u = bwd_decode(p, ui);
        for (int s = 0; s < u.T; ++s, ++it) {
            int h, m;
            bwd_step(p, u, s, h, m);
            if (!warp_wait<true, true>(bar(C::B_DQ_FULL), it & 1u, ctl, W_BWD_DQ_FULL)) return;
            tc_fence_after();
            // the whole dQ^T row of this thread's head dim, then TMEM is released (the
            // next dP^T waits for it) before any reduction is issued
            uint32_t r[128];  // r[i] = dQ^T[dim t][query i] of this block
            tmem_ld128_split(tmem + lane_off + C::T_DP, r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DQ_EMPTY));
            // lanes hold consecutive dims, so each warp-wide reduction covers 128
            // contiguous bytes of one accumulator row
            float* dst = p.dqacc + ((static_cast<size_t>(u.b) * p.Hq + h) * p.Sq_pad + m * 128) * C::D + t;
            red_rows<C::D * 4>(dst, r, std::make_index_sequence<128>{});
        }
    }
}

// ---- MMA issuer ------------------------------------------------------------------
template <bool BF16>
__device__ void bwd_mma(const BwdParams& p, uint32_t tmem, uint32_t base, uint32_t bars, CtaCtl* ctl)
{
    using C = BwdCfg<BF16>;
    using I = Issuer<C::WARP_ISSUE, true, true>;
    auto bar = [&](int i) { return bars + 8u * i; };
    uint32_t it = 0, unit_it = 0, dq_issued = 0;
    // Descriptors are built once; each MMA adds a constant byte offset / 16 to the
    // start-address field (addresses stay below 256 KB, so it cannot carry).
    const uint64_t kK = sdesc_sw128(base + C::OFF_K, 16, 1024);      // K, K-major
    const uint64_t kV = sdesc_sw128(base + C::OFF_V, 16, 1024);      // V, K-major
    const uint64_t mK = sdesc_sw128(base + C::OFF_K, 16384, 1024);   // K, MN-major
    const uint64_t kQ = sdesc_sw128(base + C::OFF_Q, 16, 1024);      // Q stage 0, K-major
    const uint64_t mQ = sdesc_sw128(base + C::OFF_Q, 16384, 1024);   // Q stage 0, MN-major
    const uint64_t kDO = sdesc_sw128(base + C::OFF_DO, 16, 1024);
    const uint64_t mDO = sdesc_sw128(base + C::OFF_DO, 16384, 1024);
    const uint64_t kDS = sdesc_sw128(base + C::OFF_DS, 16, 1024);    // dS^T, K-major
    const uint64_t mDS = sdesc_sw128(base + C::OFF_DS, 16384, 1024); // dS^T, MN-major
    constexpr uint64_t STAGE = C::TILE >> 4;
    // S^T (or dP^T) = A B^T over d, both K-major tiles
    auto mma_kk = [&](uint32_t d_t, uint64_t a, uint64_t b) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;
            I::ss(tmem + d_t, a + off, b + off, C::IDESC_KK, kk > 0);
        }
    };
    auto wait_dq_free = [&]() -> bool {
        if (dq_issued == 0) return true;
        return I::wait(bar(C::B_DQ_EMPTY), (dq_issued - 1u) & 1u, ctl, W_BWD_DQ_EMPTY);
    };
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        const BwdUnit u = bwd_decode(p, ui);
        if (u.T == 0) continue;
        if (!I::wait(bar(C::B_KV_FULL), unit_it & 1u, ctl, W_BWD_KV_FULL)) return;
        tc_fence_after();
        {
            const int st = it & 1;
            if (!I::wait(bar(C::B_Q_FULL + st), (it >> 1) & 1u, ctl, W_BWD_Q_FULL)) return;
            tc_fence_after();
            mma_kk(C::T_S, kK, kQ + st * STAGE);
            I::commit(bar(C::B_S_FULL));
            if (!wait_dq_free()) return;
            if (!I::wait(bar(C::B_DO_FULL + st), (it >> 1) & 1u, ctl, W_BWD_DO_FULL)) return;
            tc_fence_after();
            mma_kk(C::T_DP, kV, kDO + st * STAGE);
            I::commit(bar(C::B_DP_FULL));
        }
        for (int s = 0; s < u.T; ++s, ++it) {
            const int st = it & 1;
            const uint64_t mQs = mQ + st * STAGE, mDOs = mDO + st * STAGE;
            // dV += P^T dO
            if (!I::wait(bar(C::B_P_FULL), it & 1u, ctl, W_BWD_P_FULL)) return;
            tc_fence_after();
            // P^T of query half h sits at columns 64 h .. 64 h + 31 (16-bit pairs)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                I::ts(tmem + C::T_DV, tmem + C::T_S + (kk >> 2) * 64 + (kk & 3) * 8, mDOs + kk * 128u,
                       C::IDESC_KM, (s > 0 || kk > 0) ? 1u : 0u);
            I::commit(bar(C::B_DO_EMPTY + st));
            // next S^T as soon as P^T has been consumed (in-order tensor pipe)
            const int nst = (it + 1) & 1;
            if (s + 1 < u.T) {
                if (!I::wait(bar(C::B_Q_FULL + nst), ((it + 1) >> 1) & 1u, ctl, W_BWD_Q_FULL)) return;
                tc_fence_after();
                mma_kk(C::T_S, kK, kQ + nst * STAGE);
                I::commit(bar(C::B_S_FULL));
            }
            // dQ^T = K^T dS^T first (head dims on the TMEM lanes, both operands
            // MN-major), so its drain -- which gates the next dP^T -- overlaps dK
            if (!I::wait(bar(C::B_DS_FULL), it & 1u, ctl, W_BWD_DS_FULL)) return;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                I::ss(tmem + C::T_DP, mK + kk * 128u, mDS + kk * 128u, C::IDESC_MM, kk > 0 ? 1u : 0u);
            I::commit(bar(C::B_DQ_FULL));
            ++dq_issued;
            // dK += dS^T Q
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;
                I::ss(tmem + C::T_DK, kDS + off, mQs + kk * 128u, C::IDESC_KM,
                       (s > 0 || kk > 0) ? 1u : 0u);
            }
            I::commit(bar(C::B_Q_EMPTY + st));
            I::commit(bar(C::B_DS_EMPTY));
            // next dP^T once the dQ readers have drained TMEM
            if (s + 1 < u.T) {
                if (!wait_dq_free()) return;
                if (!I::wait(bar(C::B_DO_FULL + nst), ((it + 1) >> 1) & 1u, ctl, W_BWD_DO_FULL)) return;
                tc_fence_after();
                mma_kk(C::T_DP, kV, kDO + nst * STAGE);
                I::commit(bar(C::B_DP_FULL));
            }
        }
        I::commit(bar(C::B_KV_EMPTY));
        I::commit(bar(C::B_DKV_FINAL));
        ++unit_it;
    }
}

// ---- TMA producer --------------------------------------------------------------------
template <bool BF16>
struct BwdLoad {
    using C = BwdCfg<BF16>;
    const CUtensorMap *tmQ, *tmK, *tmV, *tmDO;
    uint32_t base, bars;
    CtaCtl* ctl;
    int kv_round = -1;
    int q_round[2] = {-1, -1};
    int do_round[2] = {-1, -1};

    __device__ uint32_t bar(int i) const { return bars + 8u * i; }
    __device__ void tile(uint32_t dst, const CUtensorMap* tm, uint32_t b_, int h, int row, int b)
    {
        tma_load_4d(dst, tm, b_, 0, h, row, b);
        tma_load_4d(dst + 16384u, tm, b_, 64, h, row, b);
    }
    __device__ void run(const BwdParams& p)
    {
        uint32_t it = 0, unit_it = 0;
        for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
            const BwdUnit u = bwd_decode(p, ui);
            if (u.T == 0) continue;
            if (!wait_bar_inl(bar(C::B_KV_EMPTY), (unit_it & 1u) ^ 1u, ctl, W_BWD_KV_EMPTY)) return;
            mbar_arrive_expect_tx(bar(C::B_KV_FULL), 2 * C::TILE);
            tile(base + C::OFF_K, tmK, bar(C::B_KV_FULL), u.hkv, u.k_base + u.n * 128, u.tb);
            tile(base + C::OFF_V, tmV, bar(C::B_KV_FULL), u.hkv, u.k_base + u.n * 128, u.tb);
            kv_round = static_cast<int>(unit_it);
            ++unit_it;
            for (int s = 0; s < u.T; ++s, ++it) {
                int h, m;
                bwd_step(p, u, s, h, m);
                const int st = it & 1;
                const uint32_t ph = ((it >> 1) & 1u) ^ 1u;
                if (!wait_bar_inl(bar(C::B_Q_EMPTY + st), ph, ctl, W_BWD_Q_EMPTY)) return;
                mbar_arrive_expect_tx(bar(C::B_Q_FULL + st), C::TILE + C::ROWS_BYTES);
                tile(base + C::OFF_Q + st * C::TILE, tmQ, bar(C::B_Q_FULL + st), h, u.q_base + m * 128, u.tb);
                {
                    const size_t rb = (static_cast<size_t>(u.b) * p.Hq + h) * p.Sq_pad +
                                      static_cast<size_t>(m) * 128;
                    const uint32_t dst = base + C::OFF_ROWS + st * C::ROWS_BYTES;
                    bulk_load(dst, p.L2 + rb, 512, bar(C::B_Q_FULL + st));
                    bulk_load(dst + 512, p.Dv + rb, 512, bar(C::B_Q_FULL + st));
                }
                q_round[st] = static_cast<int>(it >> 1);
                if (!wait_bar_inl(bar(C::B_DO_EMPTY + st), ph, ctl, W_BWD_DO_EMPTY)) return;
                mbar_arrive_expect_tx(bar(C::B_DO_FULL + st), C::TILE);
                tile(base + C::OFF_DO + st * C::TILE, tmDO, bar(C::B_DO_FULL + st), h, u.q_base + m * 128, u.tb);
                do_round[st] = static_cast<int>(it >> 1);
            }
        }
    }
    __device__ void drain()
    {
        const uint64_t lim = drain_limit(ctl);
        if (kv_round >= 0) drain_wait_inl(bar(C::B_KV_FULL), static_cast<uint32_t>(kv_round) & 1u, W_BWD_DRAIN, lim);
        for (int st = 0; st < 2; ++st) {
            if (q_round[st] >= 0)
                drain_wait_inl(bar(C::B_Q_FULL + st), static_cast<uint32_t>(q_round[st]) & 1u, W_BWD_DRAIN, lim);
            if (do_round[st] >= 0)
                drain_wait_inl(bar(C::B_DO_FULL + st), static_cast<uint32_t>(do_round[st]) & 1u, W_BWD_DRAIN, lim);
        }
    }
};

template <bool BF16>
__global__ void __launch_bounds__(BwdCfg<BF16>::THREADS, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const BwdParams p)
{
    using C = BwdCfg<BF16>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // swizzled TMA tiles and MMA descriptors need 1024-byte alignment
        if (threadIdx.x == 0 &&
            atomicCAS(&g_status[0], 0u, static_cast<uint32_t>(FA_ERR_UNSUPPORTED)) == 0u)
            g_status[1] = W_BWD_SMEM_ALIGN;
        return;
    }
    const uint32_t bars = base + C::OFF_BAR;
    CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem_raw + C::OFF_CTL);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        auto bar = [&](int i) { return bars + 8u * i; };
        mbar_init(bar(C::B_KV_FULL), 1);
        mbar_init(bar(C::B_KV_EMPTY), 1);
        for (int st = 0; st < 2; ++st) {
            mbar_init(bar(C::B_Q_FULL + st), 1);
            mbar_init(bar(C::B_Q_EMPTY + st), 1);
            mbar_init(bar(C::B_DO_FULL + st), 1);
            mbar_init(bar(C::B_DO_EMPTY + st), 1);
        }
        mbar_init(bar(C::B_S_FULL), 1);
        mbar_init(bar(C::B_DP_FULL), 1);
        mbar_init(bar(C::B_P_FULL), 8);
        mbar_init(bar(C::B_DS_FULL), 8);
        mbar_init(bar(C::B_DS_EMPTY), 1);
        mbar_init(bar(C::B_DQ_FULL), 1);
        mbar_init(bar(C::B_DQ_EMPTY), 4);
        mbar_init(bar(C::B_DKV_FINAL), 1);
        mbar_init(bar(C::B_DRAIN), 1);
        ctl->abort = 0u;
        ctl->wait_ns = p.wait_ns;
        fence_mbar_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_u32(&ctl->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == C::LOAD_WARP && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmDO);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    // register split (setmaxnreg, per warpgroup): warps 12-15 release registers on entry
    // to their branch, unconditionally, so the dQ warpgroup's increase always completes
    if (warp < C::DQ_WARP) {
        bwd_compute<BF16>(p, tmem, base + C::OFF_DS, base + C::OFF_ROWS, bars, ctl, warp & 3, warp >> 2);
    } else if (warp < C::MMA_WARP) {
        setmaxnreg_inc<C::REG_DQ>();  // completes once warps 12-15 have released theirs
        bwd_dq_reduce<BF16>(p, tmem, bars, ctl, warp - C::DQ_WARP);
    } else {
        setmaxnreg_dec<C::REG_CTRL>();  // all four warps, first thing, unconditionally
        if (warp == C::MMA_WARP) {
            if (C::WARP_ISSUE || lane == 0) {
                bwd_mma<BF16>(p, tmem, base, bars, ctl);
                Issuer<C::WARP_ISSUE, true, true>::commit(bars + 8u * C::B_DRAIN);
                if (lane == 0) drain_wait_inl(bars + 8u * C::B_DRAIN, 0u, W_BWD_DRAIN, drain_limit(ctl));
            }
            __syncwarp();
        } else if (warp == C::LOAD_WARP) {
            if (lane == 0) {
                BwdLoad<BF16> ld{&tmQ, &tmK, &tmV, &tmDO, base, bars, ctl};
                ld.run(p);
                ld.drain();
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::MMA_WARP) tmem_dealloc(tmem, 512);
}

}  // namespace fa
