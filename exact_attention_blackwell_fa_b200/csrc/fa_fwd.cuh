// fa_fwd.cuh -- exact attention forward for sm_100a.
//
// O = softmax(scale Q K^T [+ causal]) V and LSE, tile by tile with an online softmax
// so the score matrix never reaches HBM ("FlashAttention 4: Snellere,
// Geheugenefficiente Aandacht voor LLM's", sections "Wat is nieuw in FlashAttention
// 4", "Software-exponentials via CUDA-kernen", "Slimmere Online
// Softmax-herwaardering").  The warp roles follow the stages listed there (load,
// matrix multiply, softmax/normalise, rescale, store); the kernel design is ours:
//
//   * persistent CTAs (one per SM) walk a static list of work units
//     (batch, query head, block of query rows); units are grouped by heads so that the
//     CTAs running at the same time share K/V through L2, and for the causal mask the
//     longest units (last query blocks) go first.  Optionally (FwdParams::clc) one CTA
//     is launched per unit and the running CTAs take the others in the same order by
//     cluster launch control;
//   * one TMA thread stages Q once per unit and streams K and V through a ring of
//     shared-memory chunks (128 rows x 128 head dims, 32 KB, at d = 128 and 256; 128
//     x 64, 16 KB, at d = 192; 128-byte swizzle) guarded by full/empty mbarriers;
//   * one MMA warp issues tcgen05.mma: S = Q K^T into TMEM, then O += P V with P read
//     back from TMEM (P overwrites the first half of its own S buffer as 16-bit
//     pairs);
//   * one softmax warpgroup per Q tile (thread = one query row holding all 128 key
//     columns of a tile in registers) loads S from TMEM, applies the scale and
//     mask, keep the running row max and sum, rescale O in TMEM only when the row max
//     grew by more than kRescaleTau (log2 units), write P back into TMEM as 16-bit
//     pairs, and finally normalise and write O and LSE.  The exp2 of tiles that need
//     no mask can be split between the SFU and an FMA-pipe cubic: EMU of every four
//     pairs of exponentials on the FMA pipe (template parameter, chosen per call by
//     the host; 0 keeps every exponential on the SFU);
//
// head_dim 128: two Q tiles (256 query rows) per unit, TMEM = S0 | S1 | O0 | O1; the
// tensor core alternates between the two tiles so that one tile's softmax overlaps
// the other tile's MMAs; 384 threads, the control warpgroup handing registers to the
// softmax warpgroups (setmaxnreg).  head_dim 192 / 256: one Q tile,
// TMEM = S(a) | S(b) | O (192 / 256 columns), S double buffered so the next
// S = Q K^T runs during the softmax; each ring chunk is waited for right before and
// released right after the MMAs that read it.  head_dim 384 / 512 ("[RFC] FA4 --
// head_dim=256 & head_dim=512", Phase 4): the same one-tile pipeline, but a row's
// fp32 O no longer fits beside two S buffers, so each Q tile is two units, each
// covering one half of V's and O's head dims (TMEM = S(a) | S(b) | O half) and
// computing S = Q K^T over all of them; both units see the same scores and row
// statistics, and the first writes the LSE.
#pragma once

#include <type_traits>

#include "fa_common.cuh"

namespace fa {

// Rescale O and l only when the running row max grew by more than this (log2 units);
// until then P may reach 2^8, far inside fp32 / bf16 / fp16 range.
constexpr float kRescaleTau = 8.0f;

struct FwdParams {
    void* o;
    float* lse;
    // Packed variable-length batches (null for the dense [B, S, H, d] layout): the
    // queries of sequence b are rows cu_q[b] .. cu_q[b+1]-1 of a [total_q, Hq, d]
    // tensor, its keys rows cu_k[b] .. of [total_k, Hkv, d], of which the first
    // used_k[b] (all when used_k is null) take part.  Sq / Sk are then the maximum
    // lengths the grid is sized for.
    const int* cu_q;
    const int* cu_k;
    const int* used_k;
    int Sq_alloc;  // rows per batch entry of the q / o tensors (total_q when packed)
    // pack > 1 ("pack GQA"): the `pack` (= group) query heads of a KV head share the
    // rows of a Q tile, row r of a (batch, KV head) holding query r / pack of query
    // head kv_head * pack + r % pack; units then run over (batch, KV head)
    int pack;
    // splits > 1 (split KV, for short query sequences over long key sequences): unit u
    // covers the u-th of `splits` slices of the KV tiles and writes its O normalised by
    // its own row sums to opart [splits][B][Hq][Sq][d] and its LSE (natural log, -inf
    // for an empty slice) to lsepart [splits][B][Hq][Sq]; fa_fwd_combine_kernel merges
    int splits;
    float* opart;
    float* lsepart;
    int B, Sq, Sk, Hq, Hkv, group;
    int num_m;        // query blocks per head
    int num_tiles;    // B * Hq * num_m
    int chunk_heads;  // heads per L2 group in the unit order
    int causal;
    int inject;       // test hook: withhold the first K copy
    float sl2;        // scale * log2(e)
    // clc != 0: the grid has one CTA per unit; a running CTA takes further units by
    // cancelling CTAs that have not started (cluster launch control), in unit order.
    // clc == 0: a persistent grid walks the units with a static stride.
    int clc;
    uint64_t wait_ns;  // limit of a pipeline wait (see CtaCtl)
};

// wait-site codes reported through the device status word
enum : uint32_t {
    W_FWD_Q_FULL = 0x101, W_FWD_Q_EMPTY, W_FWD_RING_FULL, W_FWD_RING_EMPTY, W_FWD_S_FULL,
    W_FWD_P_FULL, W_FWD_O_DONE, W_FWD_O_FINAL, W_FWD_DRAIN, W_FWD_RESERVED_A, W_FWD_RESERVED_B,
    W_FWD_SMEM_ALIGN, W_FWD_SCHED_FULL, W_FWD_SCHED_EMPTY, W_FWD_CLC
};

template <int D, bool BF16>
struct FwdCfg {
    static_assert(D == 128 || D == 192 || D == 256 || D == 384 || D == 512, "head_dim");
    static constexpr int NQ = D == 128 ? 2 : 1;  // 128-row Q tiles per work unit
    static constexpr int NS = D == 128 ? 1 : 2;  // S buffers per Q tile
    // head dims of V and O a unit covers: all of them up to 256; at 384 and 512 the
    // fp32 O accumulator of a whole row (D TMEM columns) does not fit beside two S
    // buffers, so a unit covers one half of V / O (NPASS = 2 units per Q tile, each
    // recomputing S = Q K^T over all D dims)
    static constexpr int DV = D > 256 ? D / 2 : D;
    static constexpr int NPASS = D / DV;
    // ring chunk: 128 rows x CHUNK_COLS head dims (one or two 64-column swizzle atoms).
    // With one Q tile (d >= 192) each chunk is waited for just before and released
    // just after the MMAs that read it, so the ring refills while the rest of the tile
    // is still being read
    static constexpr int CHUNK_COLS = (D == 128 || D == 256) ? 128 : 64;
    static constexpr int KCH = D / CHUNK_COLS;    // chunks per K tile
    static constexpr int VCH = DV / CHUNK_COLS;   // chunks per V tile (the unit's part)
    // ring depth, in chunks: what shared memory leaves beside the Q tile
    static constexpr int NSTAGE = D == 192 ? 11 : D == 384 ? 8 : D == 512 ? 6 : 5;
    static constexpr int BM = 128;               // query rows per Q tile
    static constexpr int BN = 128;               // keys per KV tile
    // spinning waits (see fa_common.cuh) for the softmax and MMA warps
    static constexpr bool SPIN = D == 128;
    static constexpr int UNIT_ROWS = NQ * BM;
    static constexpr uint32_t CHUNK = BN * CHUNK_COLS * 2;
    static constexpr uint32_t QTILE = BM * D * 2;
    static constexpr uint32_t Q_BYTES = NQ * QTILE;
    static constexpr int SOFTMAX_WARPS = NQ * 4;     // one warpgroup per Q tile
    static constexpr int CTRL_WARP = SOFTMAX_WARPS;  // MMA warp; the TMA warp follows it
    // head_dim 128: the MMA and TMA warps plus two idle ones form a whole warpgroup,
    // which hands registers to the two softmax warpgroups (setmaxnreg); the launch
    // budget is 65536 / 384 = 168 per thread, and the host refuses to launch a build
    // whose register count differs (the increase would never be granted)
    static constexpr bool REG_SPLIT = D == 128;
    static constexpr int THREADS = (SOFTMAX_WARPS + (REG_SPLIT ? 4 : 2)) * 32;
    // (192 / 120 left the exp2-split builds spilling 84-104 bytes in the control code;
    // 184 / 136 compiles every build without spills and measured the default build
    // 2-3 % faster)
    static constexpr uint32_t REG_LAUNCH = 168, REG_SOFTMAX = 184, REG_CTRL = 136;
    static_assert(!REG_SPLIT || (THREADS == 384 && SOFTMAX_WARPS * 32 * REG_SOFTMAX + 4 * 32 * REG_CTRL <=
                                                       THREADS * REG_LAUNCH),
                  "register split exceeds the launch budget");
    static constexpr bool INL = REG_SPLIT;  // inlined waits (no calls under setmaxnreg)

    // shared memory map (offsets from the 1024-aligned dynamic shared memory base)
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_RING = Q_BYTES;
    // half-row maxima, [Q tile][step parity][half][row], then half-row sums [Q tile][half][row]
    static constexpr uint32_t OFF_BAR = OFF_RING + NSTAGE * CHUNK;
    // barrier indices
    static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1;
    static constexpr int B_FULL = 2;
    static constexpr int B_EMPTY = B_FULL + NSTAGE;
    static constexpr int B_S_FULL = B_EMPTY + NSTAGE;
    static constexpr int B_P_FULL = B_S_FULL + NQ * NS;
    static constexpr int B_O_DONE = B_P_FULL + NQ * NS;
    static constexpr int B_O_FINAL = B_O_DONE + NQ;
    static constexpr int B_DRAIN = B_O_FINAL + NQ;
    // unit schedule (clc): a ring of unit indices from the TMA thread to the softmax
    // warps and the MMA warp, and the barrier of the cancellation response
    static constexpr int NSCHED = 4;
    static constexpr int B_SCHED_FULL = B_DRAIN + 1;
    static constexpr int B_SCHED_EMPTY = B_SCHED_FULL + NSCHED;
    static constexpr int B_CLC = B_SCHED_EMPTY + NSCHED;
    static constexpr int NBAR = B_CLC + 1;
    static constexpr int SCHED_READERS = SOFTMAX_WARPS + 1;  // arrivals that free a slot
    static constexpr uint32_t OFF_CTL = OFF_BAR + 8 * NBAR;
    static constexpr uint32_t OFF_SCHED = (OFF_CTL + sizeof(CtaCtl) + 15u) & ~15u;  // int[NSCHED]
    static constexpr uint32_t OFF_CLC = OFF_SCHED + 4 * NSCHED;                      // 16-byte response
    // no alignment slack: the kernel checks that the base is 1024-byte aligned
    static constexpr uint32_t SMEM_BYTES = OFF_CLC + 16;
    static_assert(NSCHED * 4 % 16 == 0, "response alignment");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");

    // TMEM columns
    __device__ static constexpr uint32_t col_S(int q, int sb) { return NQ == 2 ? q * 128 : sb * 128; }
    __device__ static constexpr uint32_t col_O(int q) { return 256 + q * 128; }
    // P is written over the first 64 columns of its (consumed) S buffer as 16-bit
    // pairs: the packed words for keys 16 kk .. 16 kk + 15 sit at column 8 kk
    __device__ static constexpr uint32_t col_Pk(int kk) { return kk * 8; }

    static constexpr uint32_t IDESC_S = idesc_f16(BF16, 128, 128, false, false);
    static constexpr uint32_t IDESC_PV = idesc_f16(BF16, 128, CHUNK_COLS, false, true);
};

template <int UNIT_ROWS, int NPASS>
__device__ __forceinline__ void fwd_decode(const FwdParams& p, int t, int& b, int& h, int& m0, int& vpass)
{
    t /= p.splits;  // the slices of one unit are adjacent in the list
    vpass = t % NPASS;  // then the V / O parts of one Q tile
    t /= NPASS;
    const int H = p.pack > 1 ? p.Hkv : p.Hq;  // heads of the unit list
    const int BH = p.B * H;
    const int per_chunk = p.chunk_heads * p.num_m;
    const int c = t / per_chunk;
    const int r = t - c * per_chunk;
    const int first = c * p.chunk_heads;
    const int csize = min(p.chunk_heads, BH - first);
    const int mi = r / csize;
    const int bh = first + (r - mi * csize);
    const int mblk = p.causal ? (p.num_m - 1 - mi) : mi;
    b = bh / H;
    h = bh - b * H;
    m0 = mblk * UNIT_ROWS;
}

// One work unit: UNIT_ROWS query rows of one (batch entry, query head).
struct FwdUnit {
    int b, h, m0;          // h: query head (KV head when packing); m0: first row of the
                           // unit within its sequence's row space
    int R;                 // rows of that space: Sq, or Sq * pack when packing
    int tb;                // batch coordinate in the TMA maps (0 for packed sequences)
    int q_base, k_base;    // tensor row of the sequence's first query / key
    int Sq, Sk;            // the sequence's query / key counts
    int n;                 // KV tiles to visit: j0 .. j0 + n - 1
    int j0;                // first KV tile (split KV: the slice's first)
    int split;             // slice index (split KV), else 0
    int vpass;             // which part of V / O's head dims (head_dim > 256), else 0
    bool rows;             // the unit has query rows at all
};

template <int UNIT_ROWS, int NPASS>
__device__ __forceinline__ FwdUnit fwd_unit(const FwdParams& p, int t)
{
    FwdUnit u;
    fwd_decode<UNIT_ROWS, NPASS>(p, t, u.b, u.h, u.m0, u.vpass);
    if (p.cu_q != nullptr) {
        u.tb = 0;
        u.q_base = p.cu_q[u.b];
        u.k_base = p.cu_k[u.b];
        const int sq = p.cu_q[u.b + 1] - u.q_base;
        const int sk = p.used_k != nullptr ? p.used_k[u.b] : p.cu_k[u.b + 1] - u.k_base;
        u.Sq = max(0, min(sq, p.Sq));
        u.Sk = max(0, min(sk, p.Sk));
    } else {
        u.tb = u.b;
        u.q_base = 0;
        u.k_base = 0;
        u.Sq = p.Sq;
        u.Sk = p.Sk;
    }
    u.R = u.Sq * p.pack;
    u.rows = u.m0 < u.R;
    // KV tiles to visit: all of the sequence's keys, or with the causal mask (key j
    // visible to query i iff j <= i + Sk - Sq) those up to the unit's last row's limit
    const int nk = (u.Sk + 127) / 128;
    u.n = u.rows ? nk : 0;
    if (u.rows && p.causal) {
        const int last_row = (min(u.m0 + UNIT_ROWS, u.R) - 1) / p.pack;
        const long long maxcol = static_cast<long long>(last_row) + u.Sk - u.Sq;
        u.n = maxcol < 0 ? 0 : min(nk, static_cast<int>(maxcol / 128) + 1);
    }
    u.split = t % p.splits;
    u.j0 = 0;
    if (p.splits > 1) {
        const int per = (u.n + p.splits - 1) / p.splits;
        u.j0 = min(u.n, u.split * per);
        u.n = min(u.n, u.j0 + per) - u.j0;
    }
    return u;
}

// ---------------------------------------------------------------------------------
// The unit sequence one role walks.  Static: blockIdx.x, then every gridDim.x-th
// unit.  Cluster launch control: the indices the TMA thread publishes in the
// schedule ring, -1 ending it (-2: a wait gave up).  WARP: called by a whole
// converged warp (lane 0 waits and frees the slot), else by one thread.
// ---------------------------------------------------------------------------------
template <int D, bool BF16, bool WARP>
struct FwdUnits {
    using C = FwdCfg<D, BF16>;
    uint32_t bars, sched;
    CtaCtl* ctl;
    int clc;
    int t = -1;
    uint32_t k = 0;  // slots read

    __device__ int first(const FwdParams& p)
    {
        if (!clc) {
            t = blockIdx.x;
            return t < p.num_tiles ? t : -1;
        }
        return read();
    }
    __device__ int next(const FwdParams& p)
    {
        if (!clc) {
            t += gridDim.x;
            return t < p.num_tiles ? t : -1;
        }
        return read();
    }
    __device__ int read()
    {
        const uint32_t slot = k % C::NSCHED, ph = (k / C::NSCHED) & 1u;
        ++k;
        const uint32_t full = bars + 8u * (C::B_SCHED_FULL + slot);
        bool ok;
        if constexpr (WARP) ok = warp_wait<C::INL, false>(full, ph, ctl, W_FWD_SCHED_FULL);
        else ok = wait_bar_t<C::INL>(full, ph, ctl, W_FWD_SCHED_FULL);
        if (!ok) return -2;
        int v;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(sched + 4u * slot) : "memory");
        if constexpr (WARP) {
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8u * (C::B_SCHED_EMPTY + slot));
        } else {
            mbar_arrive(bars + 8u * (C::B_SCHED_EMPTY + slot));
        }
        return v;
    }
};

// ---------------------------------------------------------------------------------
// Softmax / epilogue warpgroup, one per 128-row Q tile: thread = one query row, all
// 128 key columns of a tile held in registers.
// ---------------------------------------------------------------------------------
// P = 2^x for the 32 columns cc*32 .. cc*32+31 of a tile row, packed to 16-bit pairs,
// with the row-sum partials accumulated.  SPLIT: pair j of the row goes to the FMA-pipe
// cubic when (j mod 4) < EMU, else to the SFU.
template <bool BF16, int EMU, bool SPLIT>
__device__ __forceinline__ void fwd_exp_block(const uint32_t (&sr)[128], int cc, uint64_t sl2x2, uint64_t negm2,
                                              uint64_t (&acc2)[2], uint32_t (&pk)[16])
{
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
        const int c = cc * 32 + k;
        const uint64_t x2 = ffma2(f2pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm2);
        float e0, e1;
        if (SPLIT && ((c >> 1) & 3) < EMU) {
            exp2_fma_x2(x2, e0, e1);
        } else {
            const float2 x = f2unpack(x2);
            e0 = ex2_sfu(x.x);
            e1 = ex2_sfu(x.y);
        }
        acc2[(k >> 1) & 1] = fadd2(acc2[(k >> 1) & 1], f2pack(e0, e1));
        pk[k >> 1] = pack2_p<BF16>(e0, e1);
    }
}

template <int D, bool BF16, int EMU>
__device__ void fwd_softmax_row(const FwdParams& p, uint32_t tmem, uint32_t bars, uint32_t sched, CtaCtl* ctl, int q,
                                int wq)
{
    using C = FwdCfg<D, BF16>;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const int lane = threadIdx.x & 31;
    const int r_in_tile = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::col_O(q);
    auto bar = [&](int i) { return bars + 8u * i; };
    const uint64_t sl2x2 = f2pack(p.sl2, p.sl2);
    uint32_t s_it = 0, tile_it = 0;

    FwdUnits<D, BF16, true> units{bars, sched, ctl, p.clc};
    for (int t = units.first(p); t >= 0; t = units.next(p)) {
        const FwdUnit u = fwd_unit<C::UNIT_ROWS, C::NPASS>(p, t);
        if (!u.rows) continue;  // past the end of its (shorter) sequence: nothing to do
        const int n = u.n;
        const int vr = u.m0 + q * C::BM + r_in_tile;  // this thread's row in the unit's row space
        const int row = vr / p.pack;                  // its query
        const int h = p.pack > 1 ? u.h * p.pack + (vr - row * p.pack) : u.h;
        const int q0 = (u.m0 + q * C::BM) / p.pack;   // the Q tile's first (smallest) query
        const bool row_ok = vr < u.R;
        const size_t orow_idx = static_cast<size_t>(u.tb) * p.Sq_alloc + u.q_base + row;
        // this unit's part of the O row (all of it up to head_dim 256)
        T* orow = reinterpret_cast<T*>(p.o) + (orow_idx * p.Hq + h) * D + u.vpass * C::DV;
        float* lrow = p.lse + (static_cast<size_t>(u.tb) * p.Hq + h) * p.Sq_alloc + u.q_base + row;
        // the LSE is the same for every part; the first writes it
        const bool lse_writer = u.vpass == 0;
        // split KV: this slice's partial O and LSE rows
        const size_t prow = ((static_cast<size_t>(u.split) * p.B + u.b) * p.Hq + h) * p.Sq + row;
        float* const opart_row = p.opart + prow * D + u.vpass * C::DV;
        if (n == 0 && p.splits > 1) {  // an empty slice
            if (row_ok) {
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int c = 0; c < C::DV / 4; ++c) reinterpret_cast<float4*>(opart_row)[c] = z;
                if (lse_writer) p.lsepart[prow] = -INFINITY;
            }
            continue;
        }
        if (n == 0) {  // causal with Sq > Sk (or no keys): no key is visible to any row
            if (row_ok) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c = 0; c < C::DV / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
                if (lse_writer) *lrow = -INFINITY;
            }
            continue;
        }
        // columns >= lim are masked for this row; the tile-level test uses the first
        // row of the Q tile, which has the smallest limit
        const int lim = p.causal ? min(u.Sk, row + u.Sk - u.Sq + 1) : u.Sk;
        const int lim0 = p.causal ? min(u.Sk, q0 + u.Sk - u.Sq + 1) : u.Sk;

        float m_ref = -INFINITY;  // running reference max (log2 units)
        float l = 0.0f;           // running row sum against m_ref
        for (int j = 0; j < n; ++j, ++s_it) {
            const int sb = s_it % C::NS;
            const uint32_t tS = tmem + lane_off + C::col_S(q, sb);
            if (!warp_wait<C::INL, C::SPIN>(bar(C::B_S_FULL + q * C::NS + sb), (s_it / C::NS) & 1u, ctl, W_FWD_S_FULL))
                return;
            tc_fence_after();
            uint32_t sr[128];
            {
                uint32_t (&a0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
                uint32_t (&a1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
                uint32_t (&a2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
                uint32_t (&a3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
                tmem_ld32_nowait(tS, a0);
                tmem_ld32_nowait(tS + 32, a1);
                tmem_ld32_nowait(tS + 64, a2);
                tmem_ld32_nowait(tS + 96, a3);
                tmem_wait_ld_dep(a0);
                tmem_wait_ld_dep(a1);
                tmem_wait_ld_dep(a2);
                tmem_wait_ld_dep(a3);
            }
            const int c0 = (u.j0 + j) * C::BN;  // key index of column 0
            const bool masked = c0 + C::BN > lim0;
            if (masked) {
                const int cut = lim - c0;
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= cut) sr[c] = __float_as_uint(-INFINITY);
            }
            float mx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) mx[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[4 + i]));
#pragma unroll
            for (int c = 8; c < 128; c += 8)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    mx[i] = fmax3(mx[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 4 + i]));
            const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.sl2;  // scale > 0
            const float m_new = fmaxf(m_ref, m_tile);
            const bool resc = (m_ref != -INFINITY) && (m_new - m_ref > kRescaleTau);
            const float alpha = resc ? ex2_sfu(m_ref - m_new) : 1.0f;
            if (m_ref == -INFINITY || resc) m_ref = m_new;
            // P = 2^(S scale log2e - m_ref), stored 32 columns at a time as 16-bit pairs
            // over the first 64 columns of the S buffer (every S value is in registers)
            const float negm = (m_ref == -INFINITY) ? 0.0f : -m_ref;
            const uint64_t negm2 = f2pack(negm, negm);
            uint64_t acc2[2] = {f2pack(0.0f, 0.0f), f2pack(0.0f, 0.0f)};
            // masked tiles keep every exponential on the SFU, whose 2^-inf is exactly 0
            // (the cubic's input clamp would leave 2^-126 for a masked key)
            if (EMU > 0 && !masked) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t pk[16];
                    fwd_exp_block<BF16, EMU, true>(sr, cc, sl2x2, negm2, acc2, pk);
                    tmem_st16(tS + cc * 16, pk);
                }
            } else {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t pk[16];
                    fwd_exp_block<BF16, EMU, false>(sr, cc, sl2x2, negm2, acc2, pk);
                    tmem_st16(tS + cc * 16, pk);
                }
            }
            const float2 a = f2unpack(fadd2(acc2[0], acc2[1]));
            // O must hold every earlier P V product before it is rescaled: with one S
            // buffer S_full of this tile was committed after the previous P V; with two,
            // wait for the previous P V (the MMA commits O_done after each one)
            if (__any_sync(0xffffffffu, resc)) {
                if (C::NS == 2) {
                    if (!warp_wait<C::INL, C::SPIN>(bar(C::B_O_DONE + q), (s_it - 1u) & 1u, ctl, W_FWD_O_DONE))
                        return;
                    tc_fence_after();
                }
#pragma unroll 1
                for (int cc = 0; cc < C::DV / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32_wait(tO + cc * 32, r);
#pragma unroll
                    for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
                    tmem_st32(tO + cc * 32, r);
                }
            }
            l = l * alpha + (a.x + a.y);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL + q * C::NS + sb));
        }
        // epilogue: wait for the unit's last P V, normalise and store O and LSE
        if (!warp_wait<C::INL, C::SPIN>(bar(C::B_O_FINAL + q), tile_it & 1u, ctl, W_FWD_O_FINAL)) return;
        ++tile_it;
        tc_fence_after();
        const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
        const float lse_row = (l > 0.0f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.splits > 1) {  // the slice's normalised O in fp32, and its LSE
#pragma unroll 1
            for (int cc = 0; cc < C::DV / 32; ++cc) {
                uint32_t r[32];
                tmem_ld32_wait(tO + cc * 32, r);
                if (row_ok) {
                    float4* dst = reinterpret_cast<float4*>(opart_row + cc * 32);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        dst[k] = make_float4(__uint_as_float(r[4 * k]) * inv, __uint_as_float(r[4 * k + 1]) * inv,
                                             __uint_as_float(r[4 * k + 2]) * inv, __uint_as_float(r[4 * k + 3]) * inv);
                }
            }
            if (row_ok && lse_writer) p.lsepart[prow] = lse_row;
            tc_fence_before();
            continue;
        }
#pragma unroll 1
        for (int cc = 0; cc < C::DV / 32; ++cc) {
            uint32_t r[32];
            tmem_ld32_wait(tO + cc * 32, r);
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                pk[k] = pack2<BF16>(__uint_as_float(r[2 * k]) * inv, __uint_as_float(r[2 * k + 1]) * inv);
            if (row_ok) {
                uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
                dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
            }
        }
        if (row_ok && lse_writer) *lrow = lse_row;
        tc_fence_before();
    }
}

// ---------------------------------------------------------------------------------
// MMA issuer.  head_dim 192 / 256: the whole warp runs the issue loop, converged, and each
// tcgen05 op is executed by one elected lane (warp-uniform descriptors, few
// instructions per MMA).  head_dim 128: lane 0 alone runs it (the converged form
// measured about half as fast there).
// ---------------------------------------------------------------------------------
template <int D, bool BF16>
struct FwdMma {
    using C = FwdCfg<D, BF16>;
    static constexpr bool WARP_ISSUE = D != 128;
    using I = Issuer<WARP_ISSUE, C::INL, C::SPIN>;
    uint32_t tmem, sQ, sRing, bars, sched;
    CtaCtl* ctl;
    uint32_t seq = 0;  // ring chunk sequence number

    __device__ uint32_t bar(int i) const { return bars + 8u * i; }
    __device__ bool wait(uint32_t b, uint32_t parity, uint32_t where) const { return I::wait(b, parity, ctl, where); }
    __device__ static void ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) { I::ss(d, a, b, idesc, acc); }
    __device__ static void ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) { I::ts(d, a, b, idesc, acc); }
    __device__ static void commit(uint32_t b) { I::commit(b); }
    __device__ uint32_t slot(uint32_t s) const { return sRing + (s % C::NSTAGE) * C::CHUNK; }
    __device__ bool wait_full(uint32_t s)
    {
        return wait(bar(C::B_FULL + s % C::NSTAGE), (s / C::NSTAGE) & 1u, W_FWD_RING_FULL);
    }
    __device__ void release(uint32_t s) { commit(bar(C::B_EMPTY + s % C::NSTAGE)); }

    // Descriptors are built once; every MMA then only adds a constant byte offset / 16
    // to the 14-bit start-address field (it cannot carry: addresses stay below 256 KB).
    // This keeps the single issuing thread's instruction count per MMA small -- it
    // shares its scheduler with busy softmax warps.
    uint64_t qdesc0 = 0, kdesc0 = 0, vdesc0 = 0;
    __device__ void init_descs()
    {
        qdesc0 = sdesc_sw128(sQ, 16, 1024);
        kdesc0 = sdesc_sw128(sRing, 16, 1024);
        vdesc0 = sdesc_sw128(sRing, 16384, 1024);
    }
    __device__ uint64_t slot_off(uint32_t s) const
    {
        return static_cast<uint64_t>((s % C::NSTAGE) * (C::CHUNK >> 4));
    }

    // S(q, sb) = Q_q K^T, K tile in ring chunks sK .. sK + KCH - 1.  STREAM: wait for
    // each chunk right before its k-steps and release it right after them.
    template <bool STREAM>
    __device__ bool issue_S(int q, int sb, uint32_t sK)
    {
        const uint32_t d = tmem + C::col_S(q, sb);
        const uint64_t qd = qdesc0 + static_cast<uint64_t>(q * (C::QTILE >> 4));
        uint64_t kd[C::KCH];
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) kd[c] = kdesc0 + slot_off(sK + c);
        constexpr int KPC = C::CHUNK_COLS / 16;  // k-steps per chunk
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            if constexpr (STREAM) {
                if (kk % KPC == 0) {
                    if (!wait_full(sK + kk / KPC)) return false;
                    tc_fence_after();
                }
            }
            const uint32_t aoff = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;
            const uint32_t boff = (((kk % KPC) >> 2) * 16384u + (kk & 3) * 32u) >> 4;
            ss(d, qd + aoff, kd[kk / KPC] + boff, C::IDESC_S, kk > 0);
            if constexpr (STREAM)
                if (kk % KPC == KPC - 1) release(sK + kk / KPC);
        }
        return true;
    }
    // O_q (+)= P(q, sb) V, V tile (the unit's part of its head dims) in ring chunks
    // sV .. sV + VCH - 1 (chunk c = O columns c*CHUNK_COLS .. (c+1)*CHUNK_COLS-1)
    // (k-steps 0-3 read P of key columns 0-63, 4-7 of 64-127.)  STREAM: chunk by chunk,
    // each waited for before and released after its eight k-steps.
    template <bool STREAM>
    __device__ bool issue_PV(int q, int sb, uint32_t sV, bool acc)
    {
        uint64_t vd[C::VCH];
#pragma unroll
        for (int c = 0; c < C::VCH; ++c) vd[c] = vdesc0 + slot_off(sV + c);
        const uint32_t tP = tmem + C::col_S(q, sb);
        const uint32_t tO = tmem + C::col_O(q);
        if constexpr (STREAM) {
#pragma unroll
            for (int c = 0; c < C::VCH; ++c) {
                if (!wait_full(sV + c)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ts(tO + c * C::CHUNK_COLS, tP + C::col_Pk(kk), vd[c] + (kk * 2048u >> 4), C::IDESC_PV,
                       (acc || kk > 0) ? 1u : 0u);
                release(sV + c);
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = tP + C::col_Pk(kk);
#pragma unroll
                for (int c = 0; c < C::VCH; ++c)
                    ts(tO + c * C::CHUNK_COLS, a, vd[c] + (kk * 2048u >> 4), C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
            }
        }
        return true;
    }
    __device__ bool wait_chunks(uint32_t s0)
    {
        for (int c = 0; c < C::KCH; ++c)
            if (!wait_full(s0 + c)) return false;
        tc_fence_after();
        return true;
    }
    __device__ void release_chunks(uint32_t s0)
    {
        for (int c = 0; c < C::KCH; ++c) release(s0 + c);
    }

    __device__ void run(const FwdParams& p)
    {
        uint32_t s_it[C::NQ] = {}, p_it[C::NQ] = {};
        uint32_t q_it = 0;
        FwdUnits<D, BF16, WARP_ISSUE> units{bars, sched, ctl, p.clc};
        for (int t = units.first(p); t >= 0; t = units.next(p)) {
            const int n = fwd_unit<C::UNIT_ROWS, C::NPASS>(p, t).n;
            if (n == 0) continue;
            if (!wait(bar(C::B_Q_FULL), q_it & 1u, W_FWD_Q_FULL)) return;
            ++q_it;
            tc_fence_after();
            if constexpr (C::NQ == 2) {
                // order per KV tile j: PV0(j-1), S0(j), PV1(j-1), S1(j)
                uint32_t sK = seq;
                seq += 1;
                if (!wait_chunks(sK)) return;
                for (int q = 0; q < 2; ++q) {
                    issue_S<false>(q, 0, sK);
                    commit(bar(C::B_S_FULL + q));
                    ++s_it[q];
                }
                release(sK);
                if (n == 1) commit(bar(C::B_Q_EMPTY));
                for (int j = 1; j < n; ++j) {
                    const uint32_t sV = seq;
                    seq += 1;
                    if (!wait_chunks(sV)) return;
                    if (!wait(bar(C::B_P_FULL + 0), p_it[0] & 1u, W_FWD_P_FULL)) return;
                    tc_fence_after();
                    issue_PV<false>(0, 0, sV, j > 1);
                    ++p_it[0];
                    sK = seq;
                    seq += 1;
                    if (!wait_chunks(sK)) return;
                    issue_S<false>(0, 0, sK);
                    commit(bar(C::B_S_FULL + 0));
                    ++s_it[0];
                    if (!wait(bar(C::B_P_FULL + 1), p_it[1] & 1u, W_FWD_P_FULL)) return;
                    tc_fence_after();
                    issue_PV<false>(1, 0, sV, j > 1);
                    ++p_it[1];
                    release(sV);
                    issue_S<false>(1, 0, sK);
                    commit(bar(C::B_S_FULL + 1));
                    ++s_it[1];
                    release(sK);
                    if (j == n - 1) commit(bar(C::B_Q_EMPTY));
                }
                const uint32_t sV = seq;
                seq += 1;
                if (!wait_chunks(sV)) return;
                for (int q = 0; q < 2; ++q) {
                    if (!wait(bar(C::B_P_FULL + q), p_it[q] & 1u, W_FWD_P_FULL)) return;
                    tc_fence_after();
                    issue_PV<false>(q, 0, sV, n > 1);
                    ++p_it[q];
                    commit(bar(C::B_O_FINAL + q));
                }
                release(sV);
            } else {
                // one Q tile, two S buffers; order: S(0), S(1), then per j: PV(j), S(j+2)
                for (int j = 0; j < 2 && j < n; ++j) {
                    const uint32_t sK = seq;
                    seq += C::KCH;
                    const int sb = s_it[0] & 1;
                    if (!issue_S<true>(0, sb, sK)) return;
                    commit(bar(C::B_S_FULL + sb));
                    ++s_it[0];
                }
                if (n <= 2) commit(bar(C::B_Q_EMPTY));
                for (int j = 0; j < n; ++j) {
                    const uint32_t sV = seq;
                    seq += C::VCH;
                    const int sbp = p_it[0] & 1;
                    if (!wait(bar(C::B_P_FULL + sbp), (p_it[0] >> 1) & 1u, W_FWD_P_FULL)) return;
                    tc_fence_after();
                    if (!issue_PV<true>(0, sbp, sV, j > 0)) return;
                    commit(bar(C::B_O_DONE));
                    ++p_it[0];
                    if (j + 2 < n) {
                        const uint32_t sK = seq;
                        seq += C::KCH;
                        const int sb = s_it[0] & 1;
                        if (!issue_S<true>(0, sb, sK)) return;
                        commit(bar(C::B_S_FULL + sb));
                        ++s_it[0];
                        if (j + 2 == n - 1) commit(bar(C::B_Q_EMPTY));
                    }
                }
                commit(bar(C::B_O_FINAL));
            }
        }
    }
};

// ---------------------------------------------------------------------------------
// TMA producer (one thread).  The chunk order must equal the MMA issuer's.
// ---------------------------------------------------------------------------------
template <int D, bool BF16>
struct FwdLoad {
    using C = FwdCfg<D, BF16>;
    const CUtensorMap *tmQ, *tmK, *tmV;
    uint32_t sQ, sRing, bars, sched;
    CtaCtl* ctl;
    uint32_t seq = 0;
    int filled[C::NSTAGE];  // ring round of the last fill per slot, -1 if none
    int q_round = -1;
    int inject = 0;
    uint32_t pushed = 0;    // schedule slots written
    uint32_t clc_it = 0;    // cancellation requests answered
    bool clc_pending = false;

    __device__ uint32_t bar(int i) const { return bars + 8u * i; }

    __device__ bool load_chunk(const CUtensorMap* tm, int row0, int col0, int hkv, int b)
    {
        const uint32_t s = seq++;
        const int slot = s % C::NSTAGE;
        const uint32_t round = s / C::NSTAGE;
        if (!wait_bar_t<C::INL>(bar(C::B_EMPTY + slot), (round & 1u) ^ 1u, ctl, W_FWD_RING_EMPTY)) return false;
        if (inject) {  // test hook: never fill this chunk; its consumer times out
            inject = 0;
            return true;
        }
        const uint32_t dst = sRing + slot * C::CHUNK;
        mbar_arrive_expect_tx(bar(C::B_FULL + slot), C::CHUNK);
#pragma unroll
        for (int a = 0; a < C::CHUNK_COLS / 64; ++a)
            tma_load_4d(dst + a * 16384u, tm, bar(C::B_FULL + slot), col0 + 64 * a, hkv, row0, b);
        filled[slot] = static_cast<int>(round);
        return true;
    }
    // nch chunks of one K or V tile, head dims col0 .. col0 + nch * CHUNK_COLS - 1
    __device__ bool load_kv(const CUtensorMap* tm, int row0, int hkv, int b, int nch, int col0)
    {
        for (int c = 0; c < nch; ++c)
            if (!load_chunk(tm, row0, col0 + c * C::CHUNK_COLS, hkv, b)) return false;
        return true;
    }

    // publish the next unit index (or -1) to the softmax and MMA warps
    __device__ bool push(int v)
    {
        const uint32_t slot = pushed % C::NSCHED, ph = ((pushed / C::NSCHED) & 1u) ^ 1u;
        ++pushed;
        if (!wait_bar_t<C::INL>(bar(C::B_SCHED_EMPTY + slot), ph, ctl, W_FWD_SCHED_EMPTY)) return false;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sched + 4u * slot), "r"(v) : "memory");
        mbar_arrive(bar(C::B_SCHED_FULL + slot));
        return true;
    }

    __device__ void run(const FwdParams& p)
    {
        for (int i = 0; i < C::NSTAGE; ++i) filled[i] = -1;
        inject = p.inject;
        uint32_t q_it = 0;
        const uint32_t resp = sched + 4u * C::NSCHED;  // the 16-byte cancellation response
        int t = blockIdx.x;
        if (t >= p.num_tiles) return;
        if (p.clc && !push(t)) return;
        while (true) {
            if (p.clc) {  // ask for the next unit now; the answer is read after this one's loads
                mbar_arrive_expect_tx(bar(C::B_CLC), 16);
                clc_try_cancel(resp, bar(C::B_CLC));
                clc_pending = true;
            }
            if (!load_unit(p, t, q_it)) return;
            if (p.clc) {
                if (!wait_bar_t<C::INL>(bar(C::B_CLC), clc_it & 1u, ctl, W_FWD_CLC)) return;
                clc_pending = false;
                ++clc_it;
                int x;
                t = clc_query(resp, x) ? x : -1;  // after a refusal, never ask again
                if (!push(t)) return;
                if (t < 0) return;
            } else {
                t += gridDim.x;
                if (t >= p.num_tiles) return;
            }
        }
    }

    // Q and the K / V tiles of unit t, in the MMA issuer's order; false if a wait gave up
    __device__ bool load_unit(const FwdParams& p, int t, uint32_t& q_it)
    {
        {
            const FwdUnit u = fwd_unit<C::UNIT_ROWS, C::NPASS>(p, t);
            const int n = u.n, b = u.tb;
            if (n == 0) return true;
            const int hkv = p.pack > 1 ? u.h : u.h / p.group;
            // rows past the sequence's end (the next sequence's, or out of range) are
            // loaded too: their scores are masked, their outputs never stored
            auto krow = [&](int j) { return u.k_base + (u.j0 + j) * C::BN; };
            if (!wait_bar_t<C::INL>(bar(C::B_Q_EMPTY), (q_it & 1u) ^ 1u, ctl, W_FWD_Q_EMPTY)) return false;
            mbar_arrive_expect_tx(bar(C::B_Q_FULL), C::Q_BYTES);
            // packing: one box spans the group's `pack` heads x BM / pack queries, so
            // shared-memory row r holds query r / pack of head r % pack
            const int qh = p.pack > 1 ? u.h * p.pack : u.h;
            for (int q = 0; q < C::NQ; ++q)
                for (int blk = 0; blk < D / 64; ++blk)
                    tma_load_4d(sQ + q * C::QTILE + blk * 16384u, tmQ, bar(C::B_Q_FULL), blk * 64, qh,
                                u.q_base + (u.m0 + q * C::BM) / p.pack, b);
            q_round = static_cast<int>(q_it);
            ++q_it;
            // K over all head dims; V over the unit's part of them
            const int vcol = u.vpass * C::DV;
            if constexpr (C::NQ == 2) {
                for (int j = 0; j < n; ++j) {
                    if (!load_kv(tmK, krow(j), hkv, b, C::KCH, 0)) return false;
                    if (!load_kv(tmV, krow(j), hkv, b, C::VCH, vcol)) return false;
                }
            } else {
                for (int j = 0; j < 2 && j < n; ++j)
                    if (!load_kv(tmK, krow(j), hkv, b, C::KCH, 0)) return false;
                for (int j = 0; j < n; ++j) {
                    if (!load_kv(tmV, krow(j), hkv, b, C::VCH, vcol)) return false;
                    if (j + 2 < n && !load_kv(tmK, krow(j + 2), hkv, b, C::KCH, 0)) return false;
                }
            }
        }
        return true;
    }

    // Before the CTA exits, wait for every copy this thread started (normally all
    // were consumed already and these return at once).
    __device__ void drain()
    {
        for (int i = 0; i < C::NSTAGE; ++i)
            if (filled[i] >= 0)
                drain_wait_t<C::INL>(bar(C::B_FULL + i), static_cast<uint32_t>(filled[i]) & 1u, W_FWD_DRAIN,
                                     drain_limit(ctl));
        if (q_round >= 0)
            drain_wait_t<C::INL>(bar(C::B_Q_FULL), static_cast<uint32_t>(q_round) & 1u, W_FWD_DRAIN, drain_limit(ctl));
        // an unanswered cancellation request still writes its response
        if (clc_pending) drain_wait_t<C::INL>(bar(C::B_CLC), clc_it & 1u, W_FWD_DRAIN, drain_limit(ctl));
    }
};

template <int D, bool BF16, int EMU>
__global__ void __launch_bounds__(FwdCfg<D, BF16>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p)
{
    using C = FwdCfg<D, BF16>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // swizzled TMA tiles and MMA descriptors need 1024-byte alignment
        if (threadIdx.x == 0 &&
            atomicCAS(&g_status[0], 0u, static_cast<uint32_t>(FA_ERR_UNSUPPORTED)) == 0u)
            g_status[1] = W_FWD_SMEM_ALIGN;
        return;
    }
    const uint32_t sQ = base + C::OFF_Q;
    const uint32_t sRing = base + C::OFF_RING;
    const uint32_t bars = base + C::OFF_BAR;
    const uint32_t sched = base + C::OFF_SCHED;
    CtaCtl* ctl = reinterpret_cast<CtaCtl*>(smem_raw + C::OFF_CTL);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        auto bar = [&](int i) { return bars + 8u * i; };
        mbar_init(bar(C::B_Q_FULL), 1);
        mbar_init(bar(C::B_Q_EMPTY), 1);
        for (int i = 0; i < C::NSTAGE; ++i) {
            mbar_init(bar(C::B_FULL + i), 1);
            mbar_init(bar(C::B_EMPTY + i), 1);
        }
        for (int i = 0; i < C::NQ * C::NS; ++i) {
            mbar_init(bar(C::B_S_FULL + i), 1);
            mbar_init(bar(C::B_P_FULL + i), 4);  // one arrive per softmax warp of the tile
        }
        for (int q = 0; q < C::NQ; ++q) {
            mbar_init(bar(C::B_O_DONE + q), 1);
            mbar_init(bar(C::B_O_FINAL + q), 1);
        }
        mbar_init(bar(C::B_DRAIN), 1);
        for (int i = 0; i < C::NSCHED; ++i) {
            mbar_init(bar(C::B_SCHED_FULL + i), 1);
            mbar_init(bar(C::B_SCHED_EMPTY + i), C::SCHED_READERS);
        }
        mbar_init(bar(C::B_CLC), 1);
        ctl->abort = 0u;
        ctl->wait_ns = p.wait_ns;
        fence_mbar_init();
    }
    if (warp == C::CTRL_WARP) {
        tmem_alloc(smem_u32(&ctl->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == C::CTRL_WARP + 1 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp < C::SOFTMAX_WARPS) {
        if constexpr (C::REG_SPLIT) setmaxnreg_inc<C::REG_SOFTMAX>();  // granted once warps 8-11 released theirs
        fwd_softmax_row<D, BF16, EMU>(p, tmem, bars, sched, ctl, warp / 4, warp & 3);
    } else {
        if constexpr (C::REG_SPLIT) setmaxnreg_dec<C::REG_CTRL>();  // every control warp, first thing
        if (warp == C::CTRL_WARP) {
            using M = FwdMma<D, BF16>;
            if (M::WARP_ISSUE || lane == 0) {
                M mma{tmem, sQ, sRing, bars, sched, ctl};
                mma.init_descs();
                mma.run(p);
                // all MMAs issued by this warp must finish before TMEM is released
                M::commit(bars + 8u * C::B_DRAIN);
                if (lane == 0) drain_wait_t<C::INL>(bars + 8u * C::B_DRAIN, 0u, W_FWD_DRAIN, drain_limit(ctl));
            }
            __syncwarp();
        } else if (warp == C::CTRL_WARP + 1) {
            if (lane == 0) {
                FwdLoad<D, BF16> ld{&tmQ, &tmK, &tmV, sQ, sRing, bars, sched, ctl};
                ld.run(p);
                ld.drain();
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::CTRL_WARP) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------------
// Split KV: merge the slices.  One warp per (b, h, query row): LSE = log sum_p e^LSE_p,
// O = sum_p e^(LSE_p - LSE) O_p (each O_p normalised by its own slice's row sum).
// ---------------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_fwd_combine_kernel(const FwdParams p)
{
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const long long rows = static_cast<long long>(p.B) * p.Hq * p.Sq;  // (b, h, i)
    if (row >= rows) return;
    const int i = static_cast<int>(row % p.Sq);
    const long long bh = row / p.Sq;
    const int h = static_cast<int>(bh % p.Hq), b = static_cast<int>(bh / p.Hq);
    float m = -INFINITY;
    for (int s = 0; s < p.splits; ++s) m = fmaxf(m, p.lsepart[static_cast<size_t>(s) * rows + row]);
    constexpr int PER = D / 32;  // values per lane
    float acc[PER];
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[c] = 0.0f;
    float sum = 0.0f;
    if (m != -INFINITY) {
        for (int s = 0; s < p.splits; ++s) {
            const float ls = p.lsepart[static_cast<size_t>(s) * rows + row];
            if (ls == -INFINITY) continue;
            const float w = expf(ls - m);
            sum += w;
            const float* src = p.opart + (static_cast<size_t>(s) * rows + row) * D + lane * PER;
#pragma unroll
            for (int c = 0; c < PER; c += 2) {  // 8-byte loads: PER is 4, 6 or 8
                const float2 x = *reinterpret_cast<const float2*>(src + c);
                acc[c] = fmaf(w, x.x, acc[c]);
                acc[c + 1] = fmaf(w, x.y, acc[c + 1]);
            }
        }
    }
    const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
    uint16_t* dst = static_cast<uint16_t*>(p.o) + ((static_cast<size_t>(b) * p.Sq + i) * p.Hq + h) * D + lane * PER;
    uint32_t w[PER / 2];
#pragma unroll
    for (int c = 0; c < PER / 2; ++c) w[c] = pack2<BF16>(acc[2 * c] * inv, acc[2 * c + 1] * inv);
    if constexpr (PER == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    } else if constexpr (PER == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {  // 12 bytes per lane: 4-byte aligned only
#pragma unroll
        for (int c = 0; c < PER / 2; ++c) reinterpret_cast<uint32_t*>(dst)[c] = w[c];
    }
    if (lane == 0)
        p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.Sq + i] = m == -INFINITY ? -INFINITY : m + logf(sum);
}

}  // namespace fa
