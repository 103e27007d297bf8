/*
 * attn.h - C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The operation is exact scaled dot-product attention, computed as one fused,
 * tiled kernel with an online softmax, and its recompute-based backward:
 *
 *   S = scale * Q K^T  (masked),  O = softmax_rows(S) V,  LSE_i = ln sum_j exp(S_ij)
 *
 * Sources: FlashAttention-2 overview (lshu.cn), section 2.1 (the three standard
 * steps: Q K^T, row softmax, weighted sum of V) and section 2.2 (tiled fusion,
 * online softmax with running row max m_i and row sum l_i, asynchronous
 * prefetch of the next tile); section 3.3 (the call
 * flash_attn_func(q, k, v, dropout_p, softmax_scale, causal) on tensors laid out
 * (batch, seqlen, nheads, head_dim)); section 4.2 problem 4 (causal = upper-
 * triangular mask).  The flash-attn install guide (yfxerp.com), section 1,
 * names the sliding window (window_size) and the backward that recomputes the
 * attention scores instead of storing them.
 *
 * Conventions for every entry point:
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are bfloat16 (float16 through the
 *     _ex entry points), row-major
 *     (batch, seqlen, nheads, head_dim) with head_dim contiguous and no padding
 *     between rows ("BSHD"), 16-byte aligned.  Q, O, dO, dQ have seqlen Sq;
 *     K, V, dK, dV have seqlen Sk.
 *   - lse is float32 (batch, nheads, Sq), natural-log log-sum-exp of the scaled,
 *     masked scores; -inf for a query row that sees no key (its O row is 0).
 *   - All pointers are device pointers owned by the caller; the library never
 *     allocates, frees or retains them.  Calls are asynchronous on `stream`
 *     (a cudaStream_t, may be 0 for the legacy default stream).
 *   - Arguments are validated on the host before anything is launched; on any
 *     error nothing is launched and the status says why.
 *   - Masks (delta = Sk - Sq; bounds inclusive): key j is visible to query i iff
 *       (causal == 0    or j <= i + delta)
 *       (win_left  < 0  or j >= i + delta - win_left)
 *       (win_right < 0  or j <= i + delta + win_right)
 *     -1 means "unbounded" for a window side.  Causal is aligned to the
 *     bottom-right corner when Sq != Sk.
 *   - scale must be finite and > 0 (callers wanting the default pass
 *     1/sqrt(head_dim)).
 *   - head_dim D must be 64 or 128; the dense forward and backward entry points
 *     (attn_fwd, attn_bwd, their _ex forms, the three backward stages and
 *     attn_bwd_noalloc) also take 256 (the varlen, padded and decode entry
 *     points do not).  B, H, Sq, Sk must be >= 1 and every
 *     tensor must hold fewer than 2^31 elements.
 *   - The device must be compute capability 10.0 (B200, sm_100a).
 *   - Device-side waits are bounded (about one second); a wait that runs out
 *     makes the kernel stop early, record ATTN_ERR_TIMEOUT in a device error
 *     word, release its tensor memory and return.  attn_get_last_device_error
 *     reads (and clears) that word.
 */
#ifndef EXACT_ATTENTION_156_B200_ATTN_H
#define EXACT_ATTENTION_156_B200_ATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULLPTR = 1,   /* a required pointer is NULL                         */
    ATTN_ERR_SHAPE = 2,     /* B, H, Sq or Sk < 1, a size overflows, or bad scale */
    ATTN_ERR_HEADDIM = 3,   /* head_dim not in {64, 128} (dense: {64, 128, 256})  */
    ATTN_ERR_ALIGN = 4,     /* a tensor pointer is not 16-byte aligned            */
    ATTN_ERR_WINDOW = 5,    /* win_left or win_right < -1                         */
    ATTN_ERR_ARCH = 6,      /* current device is not compute capability 10.0      */
    ATTN_ERR_DEVICE = 7,    /* a pointer is not device memory of the current GPU  */
    ATTN_ERR_LAUNCH = 8,    /* a CUDA call (descriptor build, launch) failed      */
    ATTN_ERR_TIMEOUT = 9,   /* a device-side bounded wait ran out                 */
    ATTN_ERR_WORKSPACE = 10, /* workspace NULL, misaligned or smaller than needed */
    ATTN_ERR_SCRATCH = 11,   /* problem too large for attn_bwd_noalloc's scratch  */
    ATTN_ERR_DTYPE = 12,     /* element format not one of attn_dtype              */
    ATTN_ERR_SEQLENS = 13    /* (device) malformed cu_seqlens of a packed batch   */
} attn_status;

/* Element format of the 16-bit tensors (Q, K, V, O, dO, dQ, dK, dV): the RTX
 * 5060 flash-attention page (pptc.cn), section 6.1, names fp16 and bf16 as the
 * mature input types and its section 4.4 test draws float16 tensors.
 * Accumulation is float32 in both. */
typedef enum {
    ATTN_DTYPE_BF16 = 0,
    ATTN_DTYPE_F16 = 1
} attn_dtype;

/*
 * attn_fwd - O and LSE of exact attention (FlashAttention-2 overview, section 2.2:
 * tiled fusion + online softmax; the N x N score matrix never reaches memory).
 *
 *   q   [B, Sq, H, D] bf16 (in)      k, v [B, Sk, H, D] bf16 (in)
 *   o   [B, Sq, H, D] bf16 (out)     lse  [B, H, Sq] float32 (out)
 *   scale: multiplies Q K^T; causal: 0/1; win_left, win_right: -1 or >= 0.
 * Errors: see attn_status; on error nothing is written.
 */
ATTN_API attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Sq, int Sk, int H, int D, float scale, int causal,
                     int win_left, int win_right, void* stream);

/*
 * attn_bwd_workspace_size - bytes of device workspace attn_bwd needs:
 * a float32 dQ accumulator [B, H, ceil(Sq/128)*128, D] plus two float32 row
 * vectors [B, H, ceil(Sq/128)*128] (Delta_i = sum_d dO_id O_id, and LSE in
 * base 2).  Returns 0 if the arguments are out of range.
 */
ATTN_API size_t attn_bwd_workspace_size(int B, int Sq, int H, int D);

/*
 * attn_bwd - gradients of exact attention by recomputation (flash-attn install
 * guide, section 1: the backward recomputes the scores; FlashAttention-2
 * overview, section 2.1, second anti-pattern: the standard backward re-reads
 * Q, K, V several times).  P is rebuilt from Q, K and the forward's LSE;
 *   dV = P^T dO,  dP = dO V^T,  Delta_i = rowsum(dO * O),  dS = P * (dP - Delta),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 *
 *   q, k, v, o, dout, lse: as produced/consumed by attn_fwd (in)
 *   dq [B, Sq, H, D], dk, dv [B, Sk, H, D] bf16 (out, fully overwritten)
 *   workspace: device memory of at least attn_bwd_workspace_size(B, Sq, H, D)
 *   bytes, 256-byte aligned; its contents on entry do not matter and on exit
 *   are unspecified.  Must not alias any tensor argument.
 * Errors: see attn_status; ATTN_ERR_WORKSPACE if the workspace is missing,
 * misaligned or too small.
 */
ATTN_API attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     int B, int Sq, int Sk, int H, int D, float scale, int causal,
                     int win_left, int win_right, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * The three stages attn_bwd runs, in this order on one stream, exposed so a
 * caller can place work (or timing events) between them.  Arguments mean the
 * same as in attn_bwd; the stages communicate through `workspace`.
 *
 * attn_bwd_preprocess - Delta_i = sum_d dO_id O_id (float32), the LSE in base 2,
 *   and a zeroed float32 dQ accumulator, all written into `workspace`.
 * attn_bwd_main - for every 128-key tile: recomputes P from Q, K and the
 *   workspace LSE, accumulates dV = P^T dO and dK = scale dS^T Q in tensor
 *   memory and writes them (bf16), and adds dS K into the workspace dQ
 *   accumulator with float32 bulk reduce-adds.  At head_dim 256 dK, dV and dQ
 *   are accumulated by separate tiles of one launch, and dS K is written into
 *   the accumulator whole, row by row (the preprocess then does not clear it).
 * attn_bwd_dq_finalize - dq = bf16(scale * accumulator).
 */
ATTN_API attn_status attn_bwd_preprocess(const void* o, const void* dout, const float* lse,
                                         int B, int Sq, int H, int D, void* workspace,
                                         size_t workspace_bytes, void* stream);
ATTN_API attn_status attn_bwd_main(const void* q, const void* k, const void* v, const void* dout,
                                   void* dk, void* dv, int B, int Sq, int Sk, int H, int D,
                                   float scale, int causal, int win_left, int win_right,
                                   void* workspace, size_t workspace_bytes, void* stream);
ATTN_API attn_status attn_bwd_dq_finalize(void* dq, int B, int Sq, int H, int D, float scale,
                                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * The extended forms: grouped K/V heads and the element format.
 *
 * Grouped K/V heads (GQA; MQA when Hk == 1): the pages' Transformers snippet
 * (FlashAttention-2 overview, lshu.cn, section 3.3) shapes Q with num_heads and
 * K, V with num_kv_heads for the same call.  K and V (and dK, dV) have Hk heads,
 * Q, O, dO, dQ and lse have H heads, H a multiple of Hk; query head h attends
 * with key/value head h / (H / Hk) (consecutive query heads share one K/V head).
 * dK and dV of a shared head are the sums over its query heads (accumulated in
 * the kernel, no atomics).  The workspace is sized by H, as for attn_bwd.
 *
 * dtype (attn_dtype): the format of every 16-bit tensor of the call; P and dS
 * are rounded to that format before their products, outputs are rounded from
 * float32 accumulators.
 *
 *   k, v [B, Sk, Hk, D] (in)     dk, dv [B, Sk, Hk, D] (out)
 *   every other argument as in attn_fwd / attn_bwd and its three stages.
 * Errors: as the entry points they extend; ATTN_ERR_SHAPE also if Hk < 1,
 * Hk > H or H is not a multiple of Hk; ATTN_ERR_DTYPE for an unknown dtype.
 * With Hk == H and ATTN_DTYPE_BF16 they equal attn_fwd, attn_bwd,
 * attn_bwd_preprocess, attn_bwd_main and attn_bwd_dq_finalize.
 */
ATTN_API attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int B, int Sq, int Sk, int H, int Hk, int D,
                                 int dtype, float scale, int causal, int win_left, int win_right,
                                 void* stream);
ATTN_API attn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, const float* lse, void* dq, void* dk,
                                 void* dv, int B, int Sq, int Sk, int H, int Hk, int D,
                                 int dtype, float scale, int causal, int win_left, int win_right,
                                 void* workspace, size_t workspace_bytes, void* stream);
ATTN_API attn_status attn_bwd_preprocess_ex(const void* o, const void* dout, const float* lse,
                                            int B, int Sq, int H, int D, int dtype,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);
ATTN_API attn_status attn_bwd_main_ex(const void* q, const void* k, const void* v,
                                      const void* dout, void* dk, void* dv, int B, int Sq,
                                      int Sk, int H, int Hk, int D, int dtype, float scale,
                                      int causal, int win_left, int win_right, void* workspace,
                                      size_t workspace_bytes, void* stream);
ATTN_API attn_status attn_bwd_dq_finalize_ex(void* dq, int B, int Sq, int H, int D, int dtype,
                                             float scale, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * attn_bwd_noalloc - attn_bwd for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists only for callers that
 * must not call cudaMalloc (or any allocator) at the moment they run the
 * backward, e.g. code that owns no allocator of its own inside a host that
 * manages all device memory, or latency-critical loops where an allocation
 * would implicitly synchronise the device.
 *
 * Same arguments and results as attn_bwd, without the workspace: the backward
 * scratch (the float32 dQ accumulator plus Delta and LSE rows) lives in one
 * fixed array of ATTN_NOALLOC_SCRATCH_BYTES (64 MiB) of device memory that the
 * library declares statically, so every GPU that loads the library holds it
 * until the process exits.  This call allocates nothing and calls no allocator.
 *
 *  - Problems whose backward scratch, attn_bwd_workspace_size(B, Sq, H, D),
 *    exceeds ATTN_NOALLOC_SCRATCH_BYTES are rejected with ATTN_ERR_SCRATCH
 *    before anything is launched; use attn_bwd with a workspace for those.
 *  - The first call on a device looks up the array's device address for that
 *    device (a one-time set-up per device); make that first call before any
 *    stream capture.
 *  - Every call, on every stream, shares the one array, and it keeps the last
 *    call's contents (each call re-initialises what it needs).  Calls whose
 *    execution overlaps on the GPU (concurrent streams) race on it and give
 *    wrong results: serialise them.
 *  - The looked-up address is kept for the life of the process.  The library
 *    does not survive cudaDeviceReset: a reset destroys the context that holds
 *    the array (and the library's device error word), so a process that
 *    resets a device must not call this library on that device afterwards.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
ATTN_API attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const void* dout, const float* lse, void* dq, void* dk,
                                      void* dv, int B, int Sq, int Sk, int H, int D, float scale,
                                      int causal, int win_left, int win_right, void* stream);

/*
 * attn_decode - a few new query rows per sequence against a K/V cache (the
 * pages name flash_attn_with_kvcache as the incremental-inference entry point,
 * FlashAttention-2 overview, lshu.cn, section 3.3, and give no further
 * semantics).  Sequence b attends over the first cache_seqlens[b] rows of its
 * cache (the new keys already appended by the caller); rows past that are
 * never read into the result, whatever they hold.  Causal uses the same
 * bottom-right rule: new query i (of Sq) sees keys j <= i + cache_seqlens[b] - Sq.
 * Grouped K/V heads and dtype as in the _ex entry points.
 *
 *   q             [B, Sq, H, D] (in)       k_cache, v_cache [B, Smax, Hk, D] (in)
 *   cache_seqlens [B] int32, device (in; values clamped to [0, Smax]; a row that
 *                 sees no key gets O = 0 and LSE = -inf)
 *   o             [B, Sq, H, D] (out)      lse [B, H, Sq] float32 (out)
 *   workspace     at least attn_decode_workspace_size(B, Sq, Smax, H, Hk, D) bytes,
 *                 256-byte aligned (partial results of the key splits).
 * Limits: (H / Hk) * Sq <= 128 (one K/V head's query rows form one tile).
 * Errors: as attn_fwd_ex; ATTN_ERR_SHAPE also for (H / Hk) * Sq > 128;
 * ATTN_ERR_WORKSPACE for a missing, misaligned or small workspace.
 */
ATTN_API size_t attn_decode_workspace_size(int B, int Sq, int Smax, int H, int Hk, int D);
ATTN_API attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                 const int* cache_seqlens, void* o, float* lse, int B, int Sq,
                                 int Smax, int H, int Hk, int D, int dtype, float scale,
                                 int causal, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * attn_fwd_padded / attn_bwd_padded - a padded batch: B sequences stored in
 * (B, S, H, D) tensors of one padded length, sequence b's real rows being
 * rows 0 .. seqlens[b] - 1 (the pages name the upstream padded-batch test,
 * FlashAttention-2 overview, lshu.cn, section 3.2, and say nothing more).
 * The result is that of the packed batch of the real rows (attn_fwd_varlen /
 * attn_bwd_varlen); padding rows of the inputs are never read and may hold
 * anything, non-finite values included; padding rows of the outputs are
 * written as zeros (o, dq for rows >= seqlens_q[b]; dk, dv for rows >=
 * seqlens_k[b]) and their LSE as -inf.  The real rows are gathered into
 * packed copies in the workspace, the variable-length kernels run on those,
 * and the results are scattered back.
 *
 *   q, o, dout, dq  [B, Sq, H, D]        k, v, dk, dv [B, Sk, Hk, D]
 *   lse             [B, H, Sq] float32 (out of attn_fwd_padded, in of bwd)
 *   seqlens_q / _k  [B] int32, device: 0 <= seqlens_q[b] <= Sq, 0 <= seqlens_k[b] <= Sk.
 *                   They live on the device, so they are checked there: a
 *                   length outside its range is taken as 0 (the sequence's
 *                   output rows are zeros) and the next
 *                   attn_get_last_device_error returns ATTN_ERR_SEQLENS.
 *   workspace       at least attn_fwd_padded_workspace_size / 
 *                   attn_bwd_padded_workspace_size(B, Sq, Sk, H, Hk, D) bytes,
 *                   256-byte aligned, contents ignored (0 from the size
 *                   functions means the arguments are invalid).
 * head_dim 64 or 128; grouped K/V heads and dtype as in the _ex entry points.
 * Errors: as attn_fwd_ex / attn_bwd_ex; ATTN_ERR_ALIGN if lse or a seqlens
 * pointer is not 4-byte aligned.
 */
ATTN_API size_t attn_fwd_padded_workspace_size(int B, int Sq, int Sk, int H, int Hk, int D);
ATTN_API attn_status attn_fwd_padded(const void* q, const void* k, const void* v,
                                     const int* seqlens_q, const int* seqlens_k, void* o,
                                     float* lse, int B, int Sq, int Sk, int H, int Hk, int D,
                                     int dtype, float scale, int causal, int win_left,
                                     int win_right, void* workspace, size_t workspace_bytes,
                                     void* stream);
ATTN_API size_t attn_bwd_padded_workspace_size(int B, int Sq, int Sk, int H, int Hk, int D);
ATTN_API attn_status attn_bwd_padded(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, const int* seqlens_q,
                                     const int* seqlens_k, void* dq, void* dk, void* dv, int B,
                                     int Sq, int Sk, int H, int Hk, int D, int dtype, float scale,
                                     int causal, int win_left, int win_right, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * attn_fwd_varlen / attn_bwd_varlen - a batch of B sequences of different
 * lengths packed end to end (the pages name the upstream variable-length and
 * padded-batch tests, FlashAttention-2 overview, lshu.cn, section 3.2, and say
 * nothing more).  Sequence b is rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 of
 * q, o, dout and dq and rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 of k, v, dk
 * and dv; it attends only within itself, with the causal / window rules of
 * attn_fwd applied to its own lengths (bottom-right alignment per sequence).
 * A sequence with no keys gives its rows O = 0, LSE = -inf; one with no query
 * rows gives its keys dK = dV = 0.  Grouped K/V heads and dtype as in the _ex
 * entry points.
 *
 *   q, o, dout, dq  [total_q, H, D]        k, v, dk, dv [total_k, Hk, D]
 *   lse             [H, total_q] float32 (out of attn_fwd_varlen, in of bwd)
 *   cu_seqlens_q/k  [B + 1] int32, device: cu[0] = 0, non-decreasing,
 *                   cu[B] = total; no sequence longer than max_seqlen_q / _k
 *                   (the grid is sized from the two maxima).
 *   workspace       (bwd) at least attn_bwd_varlen_workspace_size(B, total_q,
 *                   H, D) bytes, 256-byte aligned, contents ignored.
 * The boundaries live on the device, so they are checked there: a malformed
 * sequence is skipped (nothing of it read or written) and the next
 * attn_get_last_device_error returns ATTN_ERR_SEQLENS.
 * Errors: as attn_fwd_ex / attn_bwd_ex; ATTN_ERR_SHAPE also if total_q or
 * total_k < 1, or a max_seqlen is < 1 or above its total; ATTN_ERR_ALIGN if lse
 * or a cu_seqlens pointer is not 4-byte aligned.
 */
ATTN_API attn_status attn_fwd_varlen(const void* q, const void* k, const void* v,
                                     const int* cu_seqlens_q, const int* cu_seqlens_k, void* o,
                                     float* lse, int B, int total_q, int total_k,
                                     int max_seqlen_q, int max_seqlen_k, int H, int Hk, int D,
                                     int dtype, float scale, int causal, int win_left,
                                     int win_right, void* stream);
ATTN_API size_t attn_bwd_varlen_workspace_size(int B, int total_q, int H, int D);
ATTN_API attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse,
                                     const int* cu_seqlens_q, const int* cu_seqlens_k, void* dq,
                                     void* dk, void* dv, int B, int total_q, int total_k,
                                     int max_seqlen_q, int max_seqlen_k, int H, int Hk, int D,
                                     int dtype, float scale, int causal, int win_left,
                                     int win_right, void* workspace, size_t workspace_size,
                                     void* stream);

/*
 * attn_decode_split_plan - the key-split plan attn_decode uses (host logic
 * only, no device call): the cache's 128-key tiles are cut into *nsplit splits
 * of *tiles_per_split tiles, one CTA per (split, K/V head, sequence), chosen to
 * minimise ceil(CTAs / num_sms) x (tiles_per_split + 3) with at least two tiles
 * per split when the cache has more than one tile.  num_sms is the number of
 * CTAs one wave holds: attn_decode passes the current device's SM count, twice
 * that at head_dim 64 with at most 16 query rows per K/V head (two CTAs of
 * that kernel share an SM).  Errors: ATTN_ERR_NULLPTR, ATTN_ERR_SHAPE (an
 * argument < 1).
 */
ATTN_API attn_status attn_decode_split_plan(int B, int Smax, int Hk, int num_sms, int* nsplit,
                                            int* tiles_per_split);

/* attn_status_string - static English text for a status code (never NULL). */
ATTN_API const char* attn_status_string(attn_status s);

/*
 * attn_get_last_device_error - synchronises the current device, then returns
 * ATTN_ERR_TIMEOUT if a kernel of this library recorded a timed-out wait since
 * the last call, ATTN_ERR_SEQLENS if one found malformed packed-sequence
 * boundaries (and clears the record), ATTN_ERR_LAUNCH if the device reports
 * an error, ATTN_OK otherwise.
 */
ATTN_API attn_status attn_get_last_device_error(void);

/*
 * attn_device_timeout_selftest - launches one tiny kernel whose only work is
 * a bounded wait on a barrier that nothing completes, using the same bounded
 * wait as the attention kernels but with a limit of `limit_us` microseconds
 * (1..1000000).  It exercises the timeout path without faulting the GPU.
 * Returns ATTN_OK if launched; read the outcome with
 * attn_get_last_device_error (expected: ATTN_ERR_TIMEOUT).
 */
ATTN_API attn_status attn_device_timeout_selftest(int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_156_B200_ATTN_H */
