// fa_bwd_wide.cuh -- dK / dV / dQ-partials kernel of the attention backward for head_dim
// 192, 256, 384 and 512.
//
// Same arithmetic as the head_dim 128 kernel in fa_bwd.cuh (P recomputed from LSE,
// dS = P (dP - D), dV = P^T dO, dK = scale dS^T Q, dQ partials reduced in fp32), with
// a tiling that fits 256-wide heads into 512 TMEM columns and 227 KB of shared memory:
//
//   * a work unit is 64 keys of one (batch, KV head); it loops over the group's query
//     heads and 128-row query blocks;
//   * S = Q K^T and dP = dO V^T are computed query-major (M = 128 query rows, N = 64
//     keys); two compute warpgroups each own 32 of the 64 keys, a thread one query
//     row (and its LSE and D);
//   * P and dS go to shared memory as [query][key] tiles (128-byte swizzle); the
//     key-side accumulators are kept transposed, dV^T += dO^T P and dK^T += Q^T dS,
//     as two M = 128 head-dim halves each, reading dO, Q (MN-major) and P, dS
//     (MN-major) straight from the tiles already in shared memory;
//   * dQ is produced transposed, dQ^T = K^T dS^T, in two 128-dim halves into one TMEM
//     region (head dims on the lanes), each drained by the dQ warpgroup into the fp32
//     accumulator, one 128-byte segment per warp-wide reduction.
//
// head_dim 192 runs the same tiling with the fourth 64-dim block of every operand tile
// zero: it is cleared once, TMA never writes it, the d-contractions (S, dP) stop at
// dim 192, and the second head-dim half of dV^T, dK^T and dQ^T has 64 live lanes (the
// other 64 are zero and never read).
//
// head_dim 384 and 512 ("[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 4): a unit
// also carries a window of OW = D / 2 output head dims (192 or 256), and computes dV,
// dK and dQ for those dims only; the score contractions S = Q K^T and dP = dO V^T
// still run over all D dims, in two phases through the same tiles: first the other
// window's dims of Q, K, dO and V, then the unit's own, which stay in shared memory
// for the transposed products.  So every key block is visited by two units, each
// recomputing S and dP (2 x 2 of the 5 GEMMs), and K and V are loaded per phase.
//
// TMEM: S [0,64) | dP [64,128) | dQ^T half [128,256) | dV^T halves [256,384) | dK^T [384,512)
#pragma once

#include "fa_bwd.cuh"

namespace fa {

template <int DIM, bool BF16>
struct BwdWideCfg {
    static_assert(DIM == 192 || DIM == 256 || DIM == 384 || DIM == 512, "head_dim");
    static constexpr int D = DIM;
    static constexpr int OW = D > 256 ? D / 2 : D;  // output head dims per unit (window)
    static constexpr int NWIN = D / OW;             // windows per key block
    static constexpr int PH = NWIN;                 // contraction phases per step
    static constexpr int NB = OW / 64;  // 64-dim blocks loaded per operand tile
    static constexpr int BN = 64;   // keys per unit
    static constexpr int BM = 128;  // query rows per step
    // warps 0-7: compute (two warpgroups, 32 keys each), 8-11: dQ, 12: MMA, 13: TMA,
    // 14-15: idle (they complete the fourth warpgroup for setmaxnreg)
    static constexpr int THREADS = 512;
    static constexpr int DQ_WARP = 8, MMA_WARP = 12, LOAD_WARP = 13;
    // registers per thread: launched at 128; the MMA/TMA warpgroup gives 8 of them to
    // the dQ warpgroup, which then holds a whole 128-column dQ^T row in registers
    static constexpr uint32_t REG_LAUNCH = 128, REG_DQ = OW == 256 ? 136 : 144, REG_CTRL = OW == 256 ? 120 : 112;
    static_assert(8 * 32 * REG_LAUNCH + 4 * 32 * REG_DQ + 4 * 32 * REG_CTRL <= THREADS * REG_LAUNCH,
                  "register split exceeds the launch budget");
    // lane 0 of the MMA warp issues alone (the converged, elected-lane form measured
    // slower here)
    static constexpr bool WARP_ISSUE = false;
    static constexpr uint32_t KV_BLK = BN * 128;   // [64 rows][64 cols] of 16-bit values
    static constexpr uint32_t KV_BYTES = 4 * KV_BLK;  // space: four blocks
    static constexpr uint32_t Q_BLK = BM * 128;    // [128 rows][64 cols]
    static constexpr uint32_t Q_BYTES = 4 * Q_BLK;
    static constexpr uint32_t KV_LOAD = NB * KV_BLK, Q_LOAD = NB * Q_BLK;  // bytes copied
    static constexpr uint32_t PT_BYTES = BM * BN * 2;  // [128 queries][64 keys]
    static constexpr uint32_t ROWS_BYTES = 1024;       // LSE*log2(e)[128], D[128]
    static constexpr uint32_t OFF_K = 0, OFF_V = KV_BYTES, OFF_Q = 2 * KV_BYTES,
                              OFF_DO = OFF_Q + Q_BYTES, OFF_P = OFF_DO + Q_BYTES,
                              OFF_DS = OFF_P + PT_BYTES, OFF_ROWS = OFF_DS + PT_BYTES,
                              OFF_BAR = OFF_ROWS + ROWS_BYTES;
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 1, B_Q_FULL = 2, B_Q_EMPTY = 3, B_DO_FULL = 4,
                         B_DO_EMPTY = 5, B_S_FULL = 6, B_DP_FULL = 7, B_P_FULL = 8, B_P_EMPTY = 9,
                         B_DS_FULL = 10, B_DS_EMPTY = 11, B_DQ_FULL = 12, B_DQ_EMPTY = 13,
                         B_DKV_FINAL = 14, B_DRAIN = 15, B_ROWS_FULL = 16, B_ROWS_EMPTY = 17, NBAR = 18;
    static constexpr uint32_t OFF_CTL = OFF_BAR + 8 * NBAR;
    static constexpr uint32_t SMEM_BYTES = OFF_CTL + sizeof(CtaCtl);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t T_S = 0, T_DP = 64, T_DQ = 128, T_DV = 256, T_DK = 384;
    static constexpr uint32_t IDESC_S = idesc_f16(BF16, 128, 64, false, false);   // S, dP
    static constexpr uint32_t IDESC_T = idesc_f16(BF16, 128, 64, true, true);     // dV^T, dK^T
    static constexpr uint32_t IDESC_Q = idesc_f16(BF16, 128, 128, true, false);   // dQ^T half
};

enum : uint32_t {
    W_B256_KV_FULL = 0x301, W_B256_KV_EMPTY, W_B256_Q_FULL, W_B256_Q_EMPTY, W_B256_DO_FULL,
    W_B256_DO_EMPTY, W_B256_S_FULL, W_B256_DP_FULL, W_B256_P_FULL, W_B256_P_EMPTY,
    W_B256_DS_FULL, W_B256_DS_EMPTY, W_B256_DQ_FULL, W_B256_DQ_EMPTY, W_B256_DKV_FINAL,
    W_B256_DRAIN, W_B256_SMEM_ALIGN, W_B256_ROWS_FULL, W_B256_ROWS_EMPTY
};

// num_n counts 64-key blocks here; the NWIN windows of one key block are adjacent
template <int NWIN>
__device__ __forceinline__ BwdUnit bwd_wide_decode(const BwdParams& p, int t, int& win)
{
    win = t % NWIN;
    t /= NWIN;
    const int BH = p.B * p.Hkv;
    const int per_chunk = p.chunk_heads * p.num_n;
    const int c = t / per_chunk;
    const int r = t - c * per_chunk;
    const int first = c * p.chunk_heads;
    const int csize = min(p.chunk_heads, BH - first);
    const int nb = r / csize;  // causal: ascending key block = most query blocks first
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
    u.keys = u.n * 64 < u.Sk;
    const int num_m = (u.Sq + 127) / 128;
    int ms = 0;
    if (p.causal) {
        const long long imin = static_cast<long long>(u.n) * 64 - (u.Sk - u.Sq);
        ms = imin <= 0 ? 0 : static_cast<int>(imin / 128);
        if (ms > num_m) ms = num_m;
    }
    u.m_start = ms;
    u.nm = u.keys ? num_m - ms : 0;
    u.T = p.group * u.nm;
    return u;
}

// Half of a P or dS row of one query (keys 32h .. 32h+31, 16-bit) into a [128][64]
// tile, 128-byte swizzle
__device__ __forceinline__ void store_tile_half_row(uint32_t tile, int row, int half, const uint32_t (&w)[16])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t c8 = static_cast<uint32_t>(half * 4 + c);
        const uint32_t addr = tile + row * 128u + ((c8 ^ (row & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * c]),
                     "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                     : "memory");
    }
}

// ---- compute warpgroups (thread = query row, 32 keys each): P and dS; epilogue ----
template <int D, bool BF16>
__device__ void bwd_wide_compute(const BwdParams& p, uint32_t tmem, uint32_t base, uint32_t bars,
                               CtaCtl* ctl, int wq, int half)
{
    using C = BwdWideCfg<D, BF16>;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const int lane = threadIdx.x & 31;
    const int t = wq * 32 + lane;  // query row within the block, and head-dim lane later
    const int k0 = half * 32;      // this warpgroup's keys within the unit: k0 .. k0 + 31
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    auto bar = [&](int i) { return bars + 8u * i; };
    const uint64_t sl2x2 = f2pack(p.sl2, p.sl2);
    uint32_t it = 0, unit_it = 0;
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        int win;
        const BwdUnit u = bwd_wide_decode<C::NWIN>(p, ui, win);
        if (!u.keys) continue;  // past the end of its sequence's keys
        // dV^T / dK^T element of head-dim column (hf * 128 + t) of the unit's window for
        // key `key` of the unit
        auto grad_off = [&](int key, int hf) {
            return ((static_cast<size_t>(u.tb) * p.Sk_alloc + u.k_base + key) * p.Hkv + u.hkv) * C::D +
                   win * C::OW + hf * 128 + t;
        };
        if (u.T == 0) {  // keys that no query of the sequence sees: zero gradients
            T* dst = static_cast<T*>(half == 0 ? p.dv : p.dk);
            for (int key = u.n * 64; key < min(u.n * 64 + 64, u.Sk); ++key)
                for (int hf = 0; hf < 2; ++hf)
                    if (hf * 128 + t < C::OW) dst[grad_off(key, hf)] = static_cast<T>(0.0f);
            continue;
        }
        for (int s = 0; s < u.T; ++s, ++it) {
            int h, m;
            bwd_step(p, u, s, h, m);
            const int i = m * 128 + t;  // query row
            // key n*64 + c is visible iff c <= lim: (causal) c <= i + Sk - Sq - n*64, and
            // c < Sk - n*64 (rows past the sequence's keys: zeros, or the next sequence's
            // rows of a packed batch)
            const int klim = u.Sk - 1 - u.n * 64;
            const int lim = p.causal ? min(i + (u.Sk - u.Sq) - u.n * 64, klim) : klim;
            const bool masked = (p.causal && (u.n * 64 + 63 > m * 128 + u.Sk - u.Sq)) || (u.n * 64 + 64 > u.Sk);
            if (!warp_wait<true>(bar(C::B_ROWS_FULL), it & 1u, ctl, W_B256_ROWS_FULL)) return;
            float l2, dval;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(l2) : "r"(base + C::OFF_ROWS + t * 4u) : "memory");
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(dval) : "r"(base + C::OFF_ROWS + 512u + t * 4u) : "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_ROWS_EMPTY));
            const uint64_t negl2 = f2pack(-l2, -l2);
            if (!warp_wait<true>(bar(C::B_S_FULL), it & 1u, ctl, W_B256_S_FULL)) return;
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32_wait(tmem + lane_off + C::T_S + k0, r);
            float P[32];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float2 x = f2unpack(ffma2(f2pack(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2x2, negl2));
                float e0 = ex2_sfu(x.x), e1 = ex2_sfu(x.y);
                if (masked) {
                    if (k0 + c > lim) e0 = 0.0f;
                    if (k0 + c + 1 > lim) e1 = 0.0f;
                }
                P[c] = e0;
                P[c + 1] = e1;
            }
            {
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) w[k] = pack2<BF16>(P[2 * k], P[2 * k + 1]);
                if (!warp_wait<true>(bar(C::B_P_EMPTY), (it & 1u) ^ 1u, ctl, W_B256_P_EMPTY)) return;
                store_tile_half_row(base + C::OFF_P, t, half, w);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL));

            if (!warp_wait<true>(bar(C::B_DP_FULL), it & 1u, ctl, W_B256_DP_FULL)) return;
            tc_fence_after();
            tmem_ld32_wait(tmem + lane_off + C::T_DP + k0, r);
            {
                const uint64_t negd2 = f2pack(-dval, -dval);
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float2 dd = f2unpack(fadd2(f2pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), negd2));
                    w[k] = pack2<BF16>(P[2 * k] * dd.x, P[2 * k + 1] * dd.y);
                }
                if (!warp_wait<true>(bar(C::B_DS_EMPTY), (it & 1u) ^ 1u, ctl, W_B256_DS_EMPTY)) return;
                store_tile_half_row(base + C::OFF_DS, t, half, w);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DS_FULL));
        }
        // epilogue: thread t holds head-dim column (hf * 128 + t) of dV^T (half 0) or
        // dK^T (half 1)
        if (!warp_wait<true>(bar(C::B_DKV_FINAL), unit_it & 1u, ctl, W_B256_DKV_FINAL)) return;
        ++unit_it;
        tc_fence_after();
        {
            const int which = half;
            const float mul = which == 0 ? 1.0f : p.scale;
            T* dst = static_cast<T*>(which == 0 ? p.dv : p.dk);
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                if constexpr (C::OW < 256)
                    if (hf * 128 + t >= C::OW) break;  // a zero lane of the padded half
                const uint32_t col = (which == 0 ? C::T_DV : C::T_DK) + hf * 64;
                uint32_t r[32];
#pragma unroll 1
                for (int cc = 0; cc < 2; ++cc) {
                    tmem_ld32_wait(tmem + lane_off + col + cc * 32, r);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int key = u.n * 64 + cc * 32 + c;
                        if (key < u.Sk) dst[grad_off(key, hf)] = static_cast<T>(__uint_as_float(r[c]) * mul);
                    }
                }
            }
        }
        tc_fence_before();
    }
}

// ---- dQ warpgroup: two 128-dim halves of dQ^T per step -> fp32 reductions -----------
template <int D, bool BF16>
__device__ void bwd_wide_dq_reduce(const BwdParams& p, uint32_t tmem, uint32_t bars, CtaCtl* ctl, int wq)
{
    using C = BwdWideCfg<D, BF16>;
    const int lane = threadIdx.x & 31;
    const int t = wq * 32 + lane;  // head dim within the half (= TMEM lane of dQ^T)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    auto bar = [&](int i) { return bars + 8u * i; };
    uint32_t k = 0;  // dQ halves drained so far
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        int win;
        const BwdUnit u = bwd_wide_decode<C::NWIN>(p, ui, win);
        for (int s = 0; s < u.T; ++s) {
            int h, m;
            bwd_step(p, u, s, h, m);
            float* blk = p.dqacc + ((static_cast<size_t>(u.b) * p.Hq + h) * p.Sq_pad + m * 128) * C::D + t;
#pragma unroll 1
            for (int dh = 0; dh < 2; ++dh, ++k) {
                if (!warp_wait<true>(bar(C::B_DQ_FULL), k & 1u, ctl, W_B256_DQ_FULL)) return;
                if constexpr (C::OW < 256) {
                    if (dh * 128 + wq * 32 >= C::OW) {  // zero lanes of the padded half
                        if (lane == 0) mbar_arrive(bar(C::B_DQ_EMPTY));
                        continue;
                    }
                }
                tc_fence_after();
                uint32_t r[128];  // r[i] = dQ^T[dim dh*128 + t][query i]
                tmem_ld128_split(tmem + lane_off + C::T_DQ, r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_DQ_EMPTY));
                float* dst = blk + win * C::OW + dh * 128;
                red_rows<C::D * 4>(dst, r, std::make_index_sequence<128>{});
            }
        }
    }
}

// ---- MMA issuer ----------------------------------------------------------------------
template <int D, bool BF16>
__device__ void bwd_wide_mma(const BwdParams& p, uint32_t tmem, uint32_t base, uint32_t bars, CtaCtl* ctl)
{
    using C = BwdWideCfg<D, BF16>;
    using I = Issuer<C::WARP_ISSUE, true>;
    auto bar = [&](int i) { return bars + 8u * i; };
    const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sQ = base + C::OFF_Q,
                   sDO = base + C::OFF_DO, sP = base + C::OFF_P, sDS = base + C::OFF_DS;
    uint32_t it = 0, unit_it = 0, dq_issued = 0;
    // descriptors built once; each MMA adds a constant byte offset / 16 (see fa_bwd.cuh)
    const uint64_t kQ = sdesc_sw128(sQ, 16, 1024), kDO = sdesc_sw128(sDO, 16, 1024);
    const uint64_t kK = sdesc_sw128(sK, 16, 1024), kV = sdesc_sw128(sV, 16, 1024);
    const uint64_t mQ = sdesc_sw128(sQ, C::Q_BLK, 1024), mDO = sdesc_sw128(sDO, C::Q_BLK, 1024);
    const uint64_t mP = sdesc_sw128(sP, C::Q_BLK, 1024), mDS = sdesc_sw128(sDS, C::Q_BLK, 1024);
    const uint64_t kDS = sdesc_sw128(sDS, 16, 1024), mK = sdesc_sw128(sK, C::KV_BLK, 1024);
    // S (or dP) = X Y^T over d: X a [128][d] tile, Y a [64][d] tile
    auto mma_qk = [&](uint32_t d_t, uint64_t x, uint64_t y, bool acc) {
#pragma unroll
        for (int kk = 0; kk < C::OW / 16; ++kk) {
            const uint32_t xo = ((kk >> 2) * C::Q_BLK + (kk & 3) * 32u) >> 4;
            const uint32_t yo = ((kk >> 2) * C::KV_BLK + (kk & 3) * 32u) >> 4;
            I::ss(tmem + d_t, x + xo, y + yo, C::IDESC_S, (acc || kk > 0) ? 1u : 0u);
        }
    };
    // acc^T[half] (+)= X^T Z: X a [128 query][d] tile read MN-major (head-dim half
    // `hf`), Z a [128 query][64 key] tile read MN-major
    auto mma_t = [&](uint32_t d_t, uint64_t x, uint64_t z, bool acc) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                I::ss(tmem + d_t + hf * 64, x + ((2 * hf * C::Q_BLK + kk * 2048u) >> 4), z + kk * 128u,
                       C::IDESC_T, (acc || kk > 0) ? 1u : 0u);
    };
    // dQ^T half `dh` = K[:, 128 dh .. 128 dh + 127]^T dS^T: A = K read MN-major (dims
    // contiguous), B = the [query][key] dS tile read K-major
    auto mma_dq = [&](int dh) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            I::ss(tmem + C::T_DQ, mK + ((2 * dh * C::KV_BLK + kk * 2048u) >> 4), kDS + kk * 2u, C::IDESC_Q,
                   kk > 0);
    };
    auto wait_dq_free = [&]() -> bool {
        if (dq_issued == 0) return true;
        return I::wait(bar(C::B_DQ_EMPTY), (dq_issued - 1u) & 1u, ctl, W_B256_DQ_EMPTY);
    };
    if constexpr (C::PH == 1) {
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        int win;
        const BwdUnit u = bwd_wide_decode<C::NWIN>(p, ui, win);
        if (u.T == 0) continue;
        if (!I::wait(bar(C::B_KV_FULL), unit_it & 1u, ctl, W_B256_KV_FULL)) return;
        tc_fence_after();
        if (!I::wait(bar(C::B_Q_FULL), it & 1u, ctl, W_B256_Q_FULL)) return;
        tc_fence_after();
        mma_qk(C::T_S, kQ, kK, false);
        I::commit(bar(C::B_S_FULL));
        if (!I::wait(bar(C::B_DO_FULL), it & 1u, ctl, W_B256_DO_FULL)) return;
        tc_fence_after();
        mma_qk(C::T_DP, kDO, kV, false);
        I::commit(bar(C::B_DP_FULL));
        for (int s = 0; s < u.T; ++s, ++it) {
            if (!I::wait(bar(C::B_P_FULL), it & 1u, ctl, W_B256_P_FULL)) return;
            tc_fence_after();
            mma_t(C::T_DV, mDO, mP, s > 0);
            I::commit(bar(C::B_P_EMPTY));
            I::commit(bar(C::B_DO_EMPTY));
            if (!I::wait(bar(C::B_DS_FULL), it & 1u, ctl, W_B256_DS_FULL)) return;
            tc_fence_after();
            mma_t(C::T_DK, mQ, mDS, s > 0);
            I::commit(bar(C::B_Q_EMPTY));
            if (!wait_dq_free()) return;
            tc_fence_after();
            mma_dq(0);
            I::commit(bar(C::B_DQ_FULL));
            ++dq_issued;
            if (s + 1 < u.T) {
                if (!I::wait(bar(C::B_Q_FULL), (it + 1) & 1u, ctl, W_B256_Q_FULL)) return;
                tc_fence_after();
                mma_qk(C::T_S, kQ, kK, false);
                I::commit(bar(C::B_S_FULL));
                if (!I::wait(bar(C::B_DO_FULL), (it + 1) & 1u, ctl, W_B256_DO_FULL)) return;
                tc_fence_after();
                mma_qk(C::T_DP, kDO, kV, false);
                I::commit(bar(C::B_DP_FULL));
            }
            if (!wait_dq_free()) return;
            tc_fence_after();
            mma_dq(1);
            I::commit(bar(C::B_DQ_FULL));
            ++dq_issued;
            I::commit(bar(C::B_DS_EMPTY));
        }
        I::commit(bar(C::B_KV_EMPTY));
        I::commit(bar(C::B_DKV_FINAL));
        ++unit_it;
    }
    } else {
    // Two contraction phases per step: S and dP over the other window's dims, then over
    // the unit's own (whose Q, dO and K tiles the transposed products read).  K / V,
    // Q and dO each complete their FULL barrier once per phase.
    uint32_t kv_it = 0, q_it = 0, do_it = 0;
    for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
        int win;
        const BwdUnit u = bwd_wide_decode<C::NWIN>(p, ui, win);
        if (u.T == 0) continue;
        for (int s = 0; s < u.T; ++s, ++it) {
            // phase A: the other window's dims
            if (!I::wait(bar(C::B_KV_FULL), kv_it & 1u, ctl, W_B256_KV_FULL)) return;
            if (!I::wait(bar(C::B_Q_FULL), q_it & 1u, ctl, W_B256_Q_FULL)) return;
            tc_fence_after();
            mma_qk(C::T_S, kQ, kK, false);
            I::commit(bar(C::B_Q_EMPTY));
            ++q_it;
            if (!I::wait(bar(C::B_DO_FULL), do_it & 1u, ctl, W_B256_DO_FULL)) return;
            tc_fence_after();
            mma_qk(C::T_DP, kDO, kV, false);
            I::commit(bar(C::B_DO_EMPTY));
            ++do_it;
            I::commit(bar(C::B_KV_EMPTY));
            ++kv_it;
            // phase B: the unit's own window
            if (!I::wait(bar(C::B_KV_FULL), kv_it & 1u, ctl, W_B256_KV_FULL)) return;
            if (!I::wait(bar(C::B_Q_FULL), q_it & 1u, ctl, W_B256_Q_FULL)) return;
            tc_fence_after();
            mma_qk(C::T_S, kQ, kK, true);
            I::commit(bar(C::B_S_FULL));
            if (!I::wait(bar(C::B_DO_FULL), do_it & 1u, ctl, W_B256_DO_FULL)) return;
            tc_fence_after();
            mma_qk(C::T_DP, kDO, kV, true);
            I::commit(bar(C::B_DP_FULL));
            if (!I::wait(bar(C::B_P_FULL), it & 1u, ctl, W_B256_P_FULL)) return;
            tc_fence_after();
            mma_t(C::T_DV, mDO, mP, s > 0);
            I::commit(bar(C::B_P_EMPTY));
            I::commit(bar(C::B_DO_EMPTY));
            ++do_it;
            if (!I::wait(bar(C::B_DS_FULL), it & 1u, ctl, W_B256_DS_FULL)) return;
            tc_fence_after();
            mma_t(C::T_DK, mQ, mDS, s > 0);
            I::commit(bar(C::B_Q_EMPTY));
            ++q_it;
            for (int dh = 0; dh < 2; ++dh) {
                if (!wait_dq_free()) return;
                tc_fence_after();
                mma_dq(dh);
                I::commit(bar(C::B_DQ_FULL));
                ++dq_issued;
            }
            I::commit(bar(C::B_DS_EMPTY));
            I::commit(bar(C::B_KV_EMPTY));
            ++kv_it;
        }
        I::commit(bar(C::B_DKV_FINAL));
        ++unit_it;
    }
    }
}

// ---- TMA producer --------------------------------------------------------------------
template <int D, bool BF16>
struct BwdWideLoad {
    using C = BwdWideCfg<D, BF16>;
    const CUtensorMap *tmQ, *tmK, *tmV, *tmDO;  // K, V maps have 64-row boxes
    uint32_t base, bars;
    CtaCtl* ctl;
    // loads issued so far per barrier (the last one's FULL phase is drained at exit)
    uint32_t kv_n = 0, q_n = 0, do_n = 0, rows_n = 0;

    __device__ uint32_t bar(int i) const { return bars + 8u * i; }
    // K and V of the unit's 64 keys, head dims col0 .. col0 + OW - 1
    __device__ bool load_kv(const BwdUnit& u, int col0)
    {
        if (!wait_bar_inl(bar(C::B_KV_EMPTY), (kv_n & 1u) ^ 1u, ctl, W_B256_KV_EMPTY)) return false;
        mbar_arrive_expect_tx(bar(C::B_KV_FULL), 2 * C::KV_LOAD);
        for (int blk = 0; blk < C::NB; ++blk) {
            tma_load_4d(base + C::OFF_K + blk * C::KV_BLK, tmK, bar(C::B_KV_FULL), col0 + blk * 64, u.hkv,
                        u.k_base + u.n * 64, u.tb);
            tma_load_4d(base + C::OFF_V + blk * C::KV_BLK, tmV, bar(C::B_KV_FULL), col0 + blk * 64, u.hkv,
                        u.k_base + u.n * 64, u.tb);
        }
        ++kv_n;
        return true;
    }
    // the 128-row Q (or dO) tile of query head h, block m, head dims col0 .. col0 + OW - 1
    __device__ bool load_q(const CUtensorMap* tm, int full, int empty, uint32_t& n, uint32_t where,
                           const BwdUnit& u, int h, int m, int col0)
    {
        if (!wait_bar_inl(bar(empty), (n & 1u) ^ 1u, ctl, where)) return false;
        mbar_arrive_expect_tx(bar(full), C::Q_LOAD);
        const uint32_t dst = base + (full == C::B_Q_FULL ? C::OFF_Q : C::OFF_DO);
        for (int blk = 0; blk < C::NB; ++blk)
            tma_load_4d(dst + blk * C::Q_BLK, tm, bar(full), col0 + blk * 64, h, u.q_base + m * 128, u.tb);
        ++n;
        return true;
    }
    // LSE*log2(e) and D of the 128 rows of query head h, block m
    __device__ bool load_rows(const BwdParams& p, const BwdUnit& u, int h, int m)
    {
        if (!wait_bar_inl(bar(C::B_ROWS_EMPTY), (rows_n & 1u) ^ 1u, ctl, W_B256_ROWS_EMPTY)) return false;
        mbar_arrive_expect_tx(bar(C::B_ROWS_FULL), C::ROWS_BYTES);
        const size_t rb = (static_cast<size_t>(u.b) * p.Hq + h) * p.Sq_pad + static_cast<size_t>(m) * 128;
        bulk_load(base + C::OFF_ROWS, p.L2 + rb, 512, bar(C::B_ROWS_FULL));
        bulk_load(base + C::OFF_ROWS + 512, p.Dv + rb, 512, bar(C::B_ROWS_FULL));
        ++rows_n;
        return true;
    }
    __device__ void run(const BwdParams& p)
    {
        for (int rnd = 0, ui = walk_unit(0); ui < p.num_units; ui = walk_unit(++rnd)) {
            int win;
            const BwdUnit u = bwd_wide_decode<C::NWIN>(p, ui, win);
            if (u.T == 0) continue;
            if constexpr (C::PH == 1)
                if (!load_kv(u, 0)) return;
            for (int s = 0; s < u.T; ++s) {
                int h, m;
                bwd_step(p, u, s, h, m);
                // in the MMA issuer's order: per phase K / V (two phases only), Q, then
                // the rows once per step, then dO
                for (int ph = 0; ph < C::PH; ++ph) {
                    const int col0 = (C::PH == 1 ? 0 : (ph == 0 ? 1 - win : win)) * C::OW;
                    if (C::PH > 1 && !load_kv(u, col0)) return;
                    if (!load_q(tmQ, C::B_Q_FULL, C::B_Q_EMPTY, q_n, W_B256_Q_EMPTY, u, h, m, col0)) return;
                    if (ph == C::PH - 1 && !load_rows(p, u, h, m)) return;
                    if (!load_q(tmDO, C::B_DO_FULL, C::B_DO_EMPTY, do_n, W_B256_DO_EMPTY, u, h, m, col0)) return;
                }
            }
        }
    }
    __device__ void drain()
    {
        const uint64_t lim = drain_limit(ctl);
        if (kv_n) drain_wait_inl(bar(C::B_KV_FULL), (kv_n - 1u) & 1u, W_B256_DRAIN, lim);
        if (q_n) drain_wait_inl(bar(C::B_Q_FULL), (q_n - 1u) & 1u, W_B256_DRAIN, lim);
        if (do_n) drain_wait_inl(bar(C::B_DO_FULL), (do_n - 1u) & 1u, W_B256_DRAIN, lim);
        if (rows_n) drain_wait_inl(bar(C::B_ROWS_FULL), (rows_n - 1u) & 1u, W_B256_DRAIN, lim);
    }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(BwdWideCfg<D, BF16>::THREADS, 1)
    fa_bwd_dkdv_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                          const BwdParams p)
{
    using C = BwdWideCfg<D, BF16>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // swizzled TMA tiles and MMA descriptors need 1024-byte alignment
        if (threadIdx.x == 0 &&
            atomicCAS(&g_status[0], 0u, static_cast<uint32_t>(FA_ERR_UNSUPPORTED)) == 0u)
            g_status[1] = W_B256_SMEM_ALIGN;
        return;
    }
    const uint32_t bars = base + C::OFF_BAR;
    CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem_raw + C::OFF_CTL);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        auto bar = [&](int i) { return bars + 8u * i; };
        for (int i = 0; i < C::NBAR; ++i) mbar_init(bar(i), 1);
        mbar_init(bar(C::B_P_FULL), 8);
        mbar_init(bar(C::B_DS_FULL), 8);
        mbar_init(bar(C::B_DQ_EMPTY), 4);
        mbar_init(bar(C::B_ROWS_EMPTY), 8);  // one arrive per compute warp
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
    if constexpr (C::NB < 4) {
        // the fourth 64-dim block of K, V, Q and dO: zero, read by the tensor core only
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (uint32_t o = threadIdx.x * 16u; o < C::KV_BLK; o += C::THREADS * 16u) {
            *reinterpret_cast<uint4*>(smem_raw + C::OFF_K + 3 * C::KV_BLK + o) = z;
            *reinterpret_cast<uint4*>(smem_raw + C::OFF_V + 3 * C::KV_BLK + o) = z;
        }
        for (uint32_t o = threadIdx.x * 16u; o < C::Q_BLK; o += C::THREADS * 16u) {
            *reinterpret_cast<uint4*>(smem_raw + C::OFF_Q + 3 * C::Q_BLK + o) = z;
            *reinterpret_cast<uint4*>(smem_raw + C::OFF_DO + 3 * C::Q_BLK + o) = z;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    // register split (setmaxnreg, per warpgroup): warps 12-15 release registers on entry
    // to their branch, unconditionally, so the dQ warpgroup's increase always completes
    if (warp < C::DQ_WARP) {
        bwd_wide_compute<D, BF16>(p, tmem, base, bars, ctl, warp & 3, warp >> 2);
    } else if (warp < C::MMA_WARP) {
        setmaxnreg_inc<C::REG_DQ>();  // completes once warps 12-15 have released theirs
        bwd_wide_dq_reduce<D, BF16>(p, tmem, bars, ctl, warp - C::DQ_WARP);
    } else {
        setmaxnreg_dec<C::REG_CTRL>();  // all four warps, first thing, unconditionally
        if (warp == C::MMA_WARP) {
            if (C::WARP_ISSUE || lane == 0) {
                bwd_wide_mma<D, BF16>(p, tmem, base, bars, ctl);
                Issuer<C::WARP_ISSUE, true>::commit(bars + 8u * C::B_DRAIN);
                if (lane == 0) drain_wait_inl(bars + 8u * C::B_DRAIN, 0u, W_B256_DRAIN, drain_limit(ctl));
            }
            __syncwarp();
        } else if (warp == C::LOAD_WARP) {
            if (lane == 0) {
                BwdWideLoad<D, BF16> ld{&tmQ, &tmK, &tmV, &tmDO, base, bars, ctl};
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
