/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library, libfa.so.
 *
 * Operation: exact scaled-dot-product attention and its backward,
 *     O   = softmax(scale * Q K^T [+ causal mask]) V
 *     LSE = log-sum-exp of the scaled, masked scores of each query row
 * computed tile by tile with an online softmax so that the score matrix never
 * reaches device memory ("FlashAttention 4: Snellere, Geheugenefficiente Aandacht
 * voor LLM's", introduction and sections "Wat is nieuw in FlashAttention 4",
 * "Software-exponentials via CUDA-kernen", "Slimmere Online
 * Softmax-herwaardering"; the backward is listed as merged for SM100 in
 * "[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 1 table).
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, contiguous, row-major [batch, seq, heads, head_dim] in
 *     device memory ("h3-blackwell-runtime/FLASH4.md", section "API": the
 *     kernel is called in that native layout with FP16/BF16 inputs).
 *     Q, O, dO, dQ have Hq heads and Sq rows; K, V, dK, dV have Hkv heads and
 *     Sk rows.  LSE is float32 [batch, Hq, Sq] holding the natural-log
 *     log-sum-exp of scale * q.k over the visible keys (-inf for a row that sees
 *     no key).
 *   - Grouped-query attention: Hq must be a multiple of Hkv, and query head h
 *     reads key/value head h / (Hq / Hkv).
 *   - causal != 0 applies a lower-triangular mask aligned to the bottom-right
 *     corner: key j is visible to query i iff j <= i + (Sk - Sq).
 *   - head_dim d must be 128, 192, 256, 384 or 512 (192, 384, 512: "[RFC] FA4 --
 *     head_dim=256 & head_dim=512", Phase 4, symmetric head dims); dtype must be
 *     FA_BF16 or FA_FP16 and is the same for every 16-bit tensor of a call.  Every
 *     pointer must be 16-byte aligned.
 *   - Ownership: the caller owns every buffer.  The library allocates no device
 *     memory per call; scratch for the backward is the caller's workspace.
 *     Work is enqueued on `stream` and runs asynchronously; nothing synchronises.
 *   - Errors: an invalid argument returns a status and launches nothing.  There
 *     is no fallback path of any kind ("h3-blackwell-runtime/FLASH4.md": any
 *     violation raises an error instead of changing kernels).
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,    /* a size, pointer, alignment or scale is invalid          */
    FA_ERR_UNSUPPORTED = 2,    /* head_dim, dtype or GPU architecture not supported       */
    FA_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed                       */
    FA_ERR_DEVICE_TIMEOUT = 4, /* a kernel gave up on a bounded wait (see status query)   */
    FA_ERR_SCRATCH_LIMIT = 5   /* problem needs more than the built-in scratch array      */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Opaque CUDA stream handle (cudaStream_t); 0 is the legacy default stream. */
typedef void* fa_stream;

/*
 * Forward.  q [B,Sq,Hq,d], k/v [B,Sk,Hkv,d] -> o [B,Sq,Hq,d] (same dtype),
 * lse [B,Hq,Sq] float32.  scale must be finite and > 0 (1/sqrt(d) is the usual
 * choice).  Sizes: B, Sq, Sk, Hq, Hkv >= 1.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Sq, int Sk, int Hq, int Hkv, int d, int causal, float scale,
                 fa_dtype dt, fa_stream stream);

/*
 * Split-KV forward, for short query sequences over long key sequences (decode):
 * the same result as fa_fwd, with the key range of every (batch, head, query
 * block) cut into num_splits slices processed by separate CTAs, so that few query
 * rows still occupy the whole GPU; a second kernel merges the slices
 * (LSE = log sum_p e^LSE_p, O = sum_p e^(LSE_p - LSE) O_p).  num_splits <= 0 picks
 * a count from the shape and the SM count; at most 64.  With more than one slice
 * the caller provides `workspace` (256-byte aligned, at least
 * fa_fwd_splitkv_workspace_size(...) bytes, same num_splits) for the slices'
 * float32 partial O and LSE.  Layouts, dtypes and errors as fa_fwd.
 */
size_t fa_fwd_splitkv_workspace_size(int B, int Sq, int Sk, int Hq, int Hkv, int d, int num_splits);
fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                         int Sk, int Hq, int Hkv, int d, int causal, float scale, fa_dtype dt, int num_splits,
                         void* workspace, size_t workspace_bytes, fa_stream stream);

/*
 * Forward over a packed batch of variable-length sequences (the varlen row of
 * "[RFC] FA4 -- head_dim=256 & head_dim=512", Phase 1: cu_seqlens and seqused_k).
 * Sequence b's queries are rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 of
 * q [total_q, Hq, d] (o has the same layout), its keys rows cu_seqlens_k[b] ..
 * cu_seqlens_k[b+1]-1 of k, v [total_k, Hkv, d], of which the first seqused_k[b]
 * take part (seqused_k may be NULL: all of them).  lse is float32 [Hq, total_q].
 * cu_seqlens_q / cu_seqlens_k are device int32 arrays of B+1 nondecreasing offsets
 * starting at 0 and ending at total_q / total_k; seqused_k a device int32 array of
 * B counts.  max_seqlen_q / max_seqlen_k bound the sequence lengths (the grid is
 * sized by them; longer sequences are cut to them).  Each sequence is an
 * independent attention problem with the causal mask aligned to its own bottom
 * right.  Same dtypes, alignment, ownership and error behaviour as fa_fwd; the
 * offsets live on the device and are not checked by the host.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, const int* seqused_k, int B,
                        int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv,
                        int d, int causal, float scale, fa_dtype dt, fa_stream stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: the row terms
 * D = rowsum(dO * O), the log2-domain LSE copy and the float32 dQ accumulator.
 */
size_t fa_bwd_workspace_size(int B, int Sq, int Hq, int d);

/*
 * Backward.  Given the forward's inputs q, k, v, its outputs o and lse, and the
 * output gradient dO (same layout as o), writes dq [B,Sq,Hq,d], dk/dv
 * [B,Sk,Hkv,d] in the input dtype.  `workspace` is caller-owned device memory of
 * at least fa_bwd_workspace_size(B, Sq, Hq, d) bytes, 256-byte aligned; its
 * contents on entry do not matter and are overwritten.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv,
                 int B, int Sq, int Sk, int Hq, int Hkv, int d, int causal, float scale,
                 fa_dtype dt, void* workspace, size_t workspace_bytes, fa_stream stream);

/*
 * Backward over a packed batch of variable-length sequences: the inputs as for
 * fa_fwd_varlen (o, dout and dq [total_q, Hq, d]; dk, dv [total_k, Hkv, d]; lse
 * [Hq, total_q] from fa_fwd_varlen) and the workspace of
 * fa_bwd_workspace_size(B, max_seqlen_q, Hq, d).  Gradient rows of keys past
 * seqused_k[b] (allocated but not taking part) are not written; rows of keys that
 * take part but that no query sees are written as zeros.  Same ownership, ordering
 * and error behaviour as fa_bwd.
 */
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, const int* seqused_k, int B, int max_seqlen_q,
                        int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, int causal,
                        float scale, fa_dtype dt, void* workspace, size_t workspace_bytes, fa_stream stream);

/*
 * Backward that allocates nothing and takes no workspace: the same computation as
 * fa_bwd, with its scratch (the row terms and the float32 dQ accumulator) kept in a
 * fixed device array built into the library.  The paper has no counterpart to this
 * entry point; it exists for callers that cannot allocate device memory: code that
 * runs under a caller-owned memory pool or arena which forbids cudaMalloc, latency-
 * critical loops that cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree imply, and embedded hosts without a device allocator of their own.
 *
 * Limit: the scratch array is FA_NOALLOC_SCRATCH_BYTES (32 MiB) on every device
 * that loads the library, held until the process exits.  A problem whose
 * fa_bwd_workspace_size(B, Sq, Hq, d) exceeds it returns FA_ERR_SCRATCH_LIMIT and
 * launches nothing (for d = 128 that is B * Hq * ceil(Sq / 128) * 128 > 64,527
 * query rows in total).
 *
 * Set-up: the first call on each device looks up the device address of the array
 * (with that device current); make that first call before any stream capture.
 * The address is kept for the life of the process and belongs to the context that
 * was current at that first call, the device's primary context (the one the CUDA
 * runtime and PyTorch use).  Calls from another context on the same device (one
 * made with cuCtxCreate), or after cudaDeviceReset, are not supported: the library
 * is loaded into that context again and the kept address does not refer to it.
 * Every call on a device shares the one array and leaves its contents behind; the
 * kernels rewrite everything they read from it (the accumulator is zeroed by the
 * first kernel of each call), but two calls whose kernels overlap on the GPU --
 * on different streams, or from different host threads -- race on it.  Serialise
 * them.  Arguments, layouts and the other errors are as for fa_bwd.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv,
                         int B, int Sq, int Sk, int Hq, int Hkv, int d, int causal, float scale,
                         fa_dtype dt, fa_stream stream);

/*
 * exp2 split of the forward's softmax ("FlashAttention 4: Snellere,
 * Geheugenefficiente Aandacht voor LLM's", section "Software-exponentials via
 * CUDA-kernen": part of the exponentials go to a cubic polynomial on the FMA pipe
 * instead of the special-function unit; "[RFC] FA4 -- head_dim=256 &
 * head_dim=512", Phase 2 "exp2 FMA emulation": 3 of every 4 at head_dim 256).
 * pairs_of_4 in 0..3 is how many of every four pairs of exponentials of a score tile
 * use the cubic (max relative error 1.44e-4, below the 16-bit rounding of P); 0
 * keeps every exponential on the special-function unit; -1 (the initial setting)
 * selects the library's default for each head dim.  Tiles that need the causal or
 * sequence-end mask always use the special-function unit.  Process-wide; affects
 * forward launches made after the call (every forward entry point).  Any other
 * value returns FA_ERR_INVALID_ARG.
 */
fa_status fa_set_exp2_emulation(int pairs_of_4);

/* Static, human-readable name of a status code. */
const char* fa_status_string(fa_status s);

/*
 * Device-side status of the kernels run so far on this device: FA_OK, or
 * FA_ERR_DEVICE_TIMEOUT if some kernel gave up on a bounded wait (each wait in
 * the kernels gives up after the limit of fa_set_wait_timeout_ms, one second by
 * default).  Synchronises `stream` to read it.  `detail` (may be NULL) receives a
 * code naming the wait that gave up.  After a timeout the outputs of the calls
 * since the last clear are invalid; the context stays usable.
 */
fa_status fa_last_device_status(fa_stream stream, uint32_t* detail);

/* Resets the device-side status to FA_OK (enqueued on `stream`). */
fa_status fa_clear_device_status(fa_stream stream);

/*
 * Limit, in milliseconds (1 .. 600000; 1000 initially), after which a kernel's wait
 * for a pipeline stage gives up, drains what it has in flight, records
 * FA_ERR_DEVICE_TIMEOUT and returns, instead of spinning forever on a stage that
 * will not come.  The limit is measured in wall-clock time on the device, which
 * keeps running while the GPU serves another process: on a time-sliced GPU a slice
 * longer than the limit reads as a timeout, so raise it there.  Process-wide;
 * applies to launches made after the call.  Out-of-range values return
 * FA_ERR_INVALID_ARG.
 */
fa_status fa_set_wait_timeout_ms(int ms);

/*
 * Order in which the forward's CTAs take their work units ("[RFC] FA4 --
 * head_dim=256 & head_dim=512", Phase 2 "Persistent + cluster-aware tile
 * scheduler" and Phase 3 short-sequence tuning, CLC scheduling):
 *   FA_SCHED_STATIC (0): a persistent grid of at most one CTA per SM walks the
 *     units with a fixed stride (longest units first under the causal mask, heads
 *     grouped so that concurrent CTAs share K/V in L2);
 *   FA_SCHED_CLC (1): when there are more units than SMs, one CTA per unit is
 *     launched and every running CTA takes the next unit by cancelling the launch
 *     of a CTA that has not started (cluster launch control), in unit order;
 *   FA_SCHED_AUTO (2, the default): CLC for causal launches over at least 4096
 *     keys (units of unequal length, where taking the next unit when free levels
 *     the CTAs' work), STATIC otherwise.
 * Process-wide; affects launches made after the call.  Results are identical in
 * every mode.  Any other mode returns FA_ERR_INVALID_ARG.
 */
#define FA_SCHED_STATIC 0
#define FA_SCHED_CLC 1
#define FA_SCHED_AUTO 2
fa_status fa_set_unit_schedule(int mode);

/*
 * Test hook: when `mode` is 1, the next forward launch withholds its first K
 * tile copy so that the consumer's bounded wait runs out and the kernel reports
 * FA_ERR_DEVICE_TIMEOUT instead of hanging.  The hook disarms itself after one
 * launch.  0 disarms it.
 */
fa_status fa_debug_inject(int mode);

/*
 * Test hook: evaluates the kernels' base-2 exponential on `n` fp32 values.
 * `x` and `y` are device pointers to n floats (caller-owned; y may not alias x).
 * mode 0: the FMA-pipe cubic of the exp2 split ("Software-exponentials via
 * CUDA-kernen", FlashAttention 4 page: 2^x = 2^n * p(f), p our relative-minimax
 * cubic; inputs below -126 are clamped there); mode 1: the SFU instruction
 * (ex2.approx.ftz).  Enqueued on `stream`, not synchronised.  FA_ERR_INVALID_ARG
 * for n < 0, an unknown mode, or a null pointer with n > 0.
 */
fa_status fa_debug_exp2(const float* x, float* y, int n, int mode, fa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
