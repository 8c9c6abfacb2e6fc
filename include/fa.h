/*
 * fa.h -- C ABI of the B200 (sm_100a) exact IO-aware attention library
 * (libfa_b200.so).
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(scale * Q K^T + mask) V
 * ("FlashAttention (EL)", section "Problem of standard attention", the attention
 * formula) without ever writing the N x N score matrix to device memory: tiles of
 * Q, K and V are staged on chip and the softmax is applied incrementally with a
 * running row maximum and exp-sum ("FlashAttention (EL)", sections "Tiling" and
 * "Online computation of Softmax"; "Flash Attention: Ako transformery zvladaju
 * miliony tokenov", section 2).  The backward pass recomputes the probabilities
 * from the saved per-row log-sum-exp instead of storing them ("Flash Attention
 * uitgelegd: een uitgebreide gids", section "Recomputation").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major (B, H, N, d) with d innermost -- the layout of
 *    the scaled_dot_product_attention call shown on "Flash Attention: Ako
 *    transformery ...", section 6.  Per-row statistics (LSE) are (B, H, N).
 *  - Q and K/V have the same sequence length N (square problem).
 *  - causal = 1 masks key j for query i when j > i (query i sees keys 0..i, the
 *    diagonal included); causal = 0 is full (bidirectional) attention.
 *  - scale multiplies Q K^T before masking; callers normally pass 1/sqrt(d).
 *  - LSE_i = ln sum_j exp(scale * S_ij) over the visible keys (natural log of the
 *    scaled, masked scores), fp32.
 *  - Every pointer is CALLER-OWNED DEVICE memory on the current CUDA device.  The
 *    library allocates no memory and keeps no state between calls except one
 *    device-resident error word per device (see fa_last_device_status).
 *  - Value range.  The tensor-core products that need more than bf16's 8 significant
 *    bits (P V in the forward; all products of the backward) read fp16 copies of the bf16
 *    inputs.  fp16 ends at 65504, so every copy is the input times a power of two 2^e
 *    chosen from the tensor's largest magnitude (one e per tensor; per 128-key tile of V
 *    in the forward without a workspace), and the kernels undo 2^e exactly; e = 0, i.e.
 *    the plain conversion, whenever the magnitudes lie in [2^-4, 2^15].  Every finite
 *    bf16 input is therefore handled, with these limits, reported as FA_ERR_RANGE by
 *    fa_last_device_status (the outputs of the rows concerned are then unspecified):
 *    a non-finite input; a score Q K^T or a D = rowsum(dO * O) beyond the fp32 range
 *    (about max|Q| max|K| d >= 2^128); in fa_fwd / fa_fwd_gqa (no workspace), a V element of
 *    magnitude 2^31 or more.  In fa_fwd / fa_fwd_gqa V tiles are only scaled down, so V
 *    elements below 2^-14 keep fp16's subnormal grid (absolute error <= 2^-25 each).
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream) and do
 *    not synchronise.  Argument errors are detected on the host before anything
 *    is launched; nothing is written then.
 *  - B, H or N equal to 0 is an empty problem: FA_OK, nothing launched.
 *  - Supported: d in {64, 128}; d = 256 also for the forward with a workspace
 *    (fa_fwd_ws, fa_attn_fwd) and for every backward (fa_bwd, fa_bwd_gqa, fa_bwd_ws,
 *    fa_attn_bwd, fa_bwd_noalloc); the 8-bit forward takes d = 128 or 64; a
 *    B200-class GPU (compute capability 10.0).
 *
 * Thread safety: calls may be issued from several host threads; calls whose
 * work overlaps on the GPU must not share output buffers or a workspace.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad scale/causal, H not a multiple of
                             H_kv, workspace too small */
  FA_ERR_UNSUPPORTED = 2, /* head dim not supported by the call, sizes beyond limits, not a CC 10.0 device */
  FA_ERR_MISALIGNED = 3,  /* a tensor base address is not 16-byte aligned (TMA requirement) */
  FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
  FA_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait (reported by fa_last_device_status) */
  FA_ERR_RANGE = 6        /* an input beyond the value range above (reported by fa_last_device_status) */
} fa_status;

/*
 * fa_fwd -- forward pass, bf16 in / bf16 out, on tensor cores.
 *   q, k, v : const bf16 (B, H, N, d), 16-byte aligned.
 *   o       : bf16 (B, H, N, d) output, 16-byte aligned; must not alias q, k, v.
 *   lse     : fp32 (B, H, N) output (natural-log LSE, see above), or NULL to skip.
 *   B, H, N : batch, heads, sequence length (>= 0).  d: head dim, 64 or 128.
 *   scale   : finite, > 0.   causal: 0 or 1.   stream: CUDA stream.
 * Q K^T is a bf16 product with fp32 accumulation; the probabilities are rounded
 * to fp16 (round to nearest even) for the P V product, whose V operand is an fp16
 * copy of the bf16 V made on chip (each 128-key tile scaled by a power of two when its
 * magnitudes exceed 2^15, see "Value range"); the row sums are fp32; O is rounded to
 * bf16 once at the end.  The attention formula is "FlashAttention (EL)", section
 * "Problem of standard attention"; the tiled computation with an online softmax is its
 * sections "Tiling" and "Online computation of Softmax".
 * A training forward that feeds fa_bwd_gqa / fa_attn_bwd can also write the bf16
 * residual O_fp32 - O_bf16 (fa_fwd_gqa with H_kv = H, fa_fwd_ws, fa_attn_fwd): the
 * backward then forms rowsum(dO * O) from an fp32-accurate O.  Without it (fa_fwd ->
 * fa_bwd) D carries O's bf16 rounding, which costs the gradients up to ~0.2 of absolute
 * accuracy on sharply peaked softmax rows (a few keys ~8x larger than the rest).
 * Returns FA_OK once the kernel is enqueued.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                        float scale, int causal, fa_stream_t stream);

/*
 * fa_fwd_gqa -- fa_fwd for grouped-query / multi-query attention ("Flash
 * Attention: Ako transformery ...", section 5, and "FlashAttention (EL)", the list
 * of extensions, name GQA/MQA support; the grouping below is the reading taken).
 *   q, o    : (B, H, N, d) as in fa_fwd;  lse: (B, H, N).
 *   o_resid : bf16 (B, H, N, d) output or NULL: the residual O_fp32 - O_bf16 of the
 *             final rounding of O, for fa_bwd_gqa / fa_attn_bwd.
 *   k, v    : const bf16 (B, H_kv, N, d), 16-byte aligned.
 *   H_kv    : key/value heads, >= 1, H a multiple of H_kv (H_kv = 1: MQA, H_kv = H: plain
 *             multi-head attention; with o_resid = NULL identical to fa_fwd).
 * Query head h of batch entry b attends with key/value head h / (H / H_kv) of the
 * same batch entry (consecutive groups of H / H_kv query heads share one K/V head).
 * Everything else (precision, alignment, errors, asynchrony) as fa_fwd.
 */
FA_API fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, void* o_resid, int B,
                            int H, int H_kv, int N, int d, float scale, int causal, fa_stream_t stream);

/*
 * fa_fwd_workspace_size / fa_fwd_ws -- the forward pass of fa_fwd_gqa (H_kv = H for
 * plain multi-head attention) with a caller workspace, used to run the V operand's
 * bf16 -> fp16 conversion as one streaming pass before the attention kernel instead of
 * inside it (fa_fwd / fa_fwd_gqa convert each V tile on chip, on two warps that share
 * SM sub-partitions with half of the softmax warps).  Results are identical to fa_fwd_gqa
 * (every unit computes the same values in the same order) whenever V's magnitudes lie in
 * [2^-4, 2^15] (both copies unscaled; outside it the workspace copy is scaled per tensor,
 * the on-chip one per tile).
 *   workspace       : device buffer of at least fa_fwd_workspace_size(B, H_kv, N, d)
 *                     bytes (an fp16 copy V 2^e of V with one exponent e for the tensor,
 *                     a work counter and 9.5 KB of per-block maxima), 256-byte aligned,
 *                     caller-owned; contents on entry do not matter, unspecified on
 *                     return.  NULL is an error.
 * With a workspace the attention kernel is persistent (one CTA per SM taking work units
 * from the counter, so one unit's epilogue overlaps the next unit's loads and first
 * products); calls that overlap on the GPU need separate workspaces.
 *   workspace_bytes : its size.
 * fa_fwd_workspace_size returns 0 for an empty or invalid problem.  Everything else as
 * fa_fwd_gqa, except that d may also be 256 (the head dimension FlashAttention-2 added:
 * "FlashAttention (EL)", section "FlashAttention-2 (2023)"): a kernel of its own with one
 * 128-row query tile per work unit, because S and a 256-column O of two tiles do not fit in
 * tensor memory.  Every backward entry point takes d = 256 as well.
 */
FA_API size_t fa_fwd_workspace_size(int B, int H_kv, int N, int d);
FA_API fa_status fa_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, void* o_resid, int B,
                           int H, int H_kv, int N, int d, float scale, int causal, void* workspace,
                           size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_f32 -- the same forward pass on fp32 inputs and outputs, computed
 * entirely in fp32 on the CUDA cores (no input rounding).  Meant for small
 * problems and checks; same arguments and rules as fa_fwd except dtypes, and
 * pointers need only 4-byte alignment.
 */
FA_API fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N,
                     int d, float scale, int causal, fa_stream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs for this
 * problem (fp16 copies of Q, K, V, dO, two fp32 (B, H, N rounded up to 128) row
 * vectors, 256 bytes of work counters and copy exponents, 18.5 KB of per-block
 * maxima).  Returns 0 for an empty or invalid problem.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- backward pass: gradients of sum(O * dO) with respect to Q, K, V.
 *   q, k, v, o, dout : const bf16 (B, H, N, d), 16-byte aligned; o and lse are the
 *                      outputs of fa_fwd on the same q, k, v, scale and causal.
 *   lse              : const fp32 (B, H, N).
 *   dq, dk, dv       : fp32 (B, H, N, d) outputs, 16-byte aligned, not aliasing
 *                      any input.  Overwritten (not accumulated into).
 *   workspace        : device buffer of at least fa_bwd_workspace_size(B,H,N,d)
 *                      bytes (the call trusts that size: the signature carries none),
 *                      256-byte aligned, caller-owned; its contents on entry do not
 *                      matter and on return are unspecified.
 * The probabilities are recomputed from LSE ("Flash Attention uitgelegd: een
 * uitgebreide gids", section "Recomputation"); the gradients follow from the softmax
 * Jacobian.  The tensor-core products run in fp16 on copies x 2^e of the bf16 inputs
 * (one exponent per tensor, see "Value range"), with fp32 accumulation; gradients are
 * fp32.  rowsum(dO * O) uses the bf16 O (see fa_fwd for the residual variant).
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, float* dq, float* dk, float* dv, int B, int H, int N, int d, float scale,
                        int causal, void* workspace, fa_stream_t stream);

/*
 * fa_bwd_gqa_workspace_size / fa_bwd_gqa -- fa_bwd for grouped-query attention
 * (grouping as in fa_fwd_gqa).
 *   q, o, dout, dq          : (B, H, N, d);  lse: (B, H, N).
 *   o_resid                 : const bf16 (B, H, N, d) residual from the forward, or NULL
 *                             (then rowsum(dO * O) uses the bf16 O alone: less accurate).
 *   k, v                    : const bf16 (B, H_kv, N, d).
 *   dk, dv                  : fp32 (B, H_kv, N, d) outputs: the gradient of a shared
 *                             key/value head is the sum over the query heads of its
 *                             group.  Overwritten (not accumulated into).
 *   workspace               : at least fa_bwd_gqa_workspace_size(B, H, H_kv, N, d)
 *                             bytes (fp16 copies of Q and dO with H heads, of K and
 *                             V with H_kv heads, the two fp32 row vectors and, when
 *                             B * H_kv * ceil(N / 128) < 592, fp32 partial dK and dV
 *                             for the CTAs that split a group's query heads; their
 *                             sum is formed in a fixed order: results are
 *                             deterministic).
 *   workspace_bytes         : its size.
 * With H_kv = H and o_resid = NULL both are identical to fa_bwd_workspace_size / fa_bwd.
 * Everything else as fa_bwd.
 */
FA_API size_t fa_bwd_gqa_workspace_size(int B, int H, int H_kv, int N, int d);
FA_API fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                            const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H,
                            int H_kv, int N, int d, float scale, int causal, void* workspace,
                            size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_ws_workspace_size / fa_bwd_ws -- fa_bwd_gqa that reuses the fp16 copy of V which
 * fa_fwd_ws left in its workspace, instead of converting V again (the backward's streaming
 * preprocess then reads and writes 4 bytes fewer per element of V).
 *   fwd_workspace, fwd_workspace_bytes : the workspace of the fa_fwd_ws call that produced
 *                             o (and o_resid, lse) from this v, with the same B, H_kv, N,
 *                             d, unchanged since (no other forward in it); 256-byte
 *                             aligned, at least fa_fwd_workspace_size(B, H_kv, N, d)
 *                             bytes.  The backward may rewrite the V copy there (and the
 *                             exponent recorded with it) when the bound on the fp16 dS
 *                             asks for another power-of-two scaling of V than the copy
 *                             holds (see "Value range"): a later fa_bwd_ws on the same
 *                             forward workspace stays correct.
 *   workspace                : at least fa_bwd_ws_workspace_size(B, H, H_kv, N, d) bytes
 *                             (fa_bwd_gqa's workspace without the V copy).
 * Everything else as fa_bwd_gqa; the gradients are identical to fa_bwd_gqa's.
 * Errors: FA_ERR_INVALID_ARG for a NULL or too small forward workspace,
 * FA_ERR_MISALIGNED for one not 256-byte aligned; otherwise as fa_bwd_gqa.
 */
FA_API size_t fa_bwd_ws_workspace_size(int B, int H, int H_kv, int N, int d);
FA_API fa_status fa_bwd_ws(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                           const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H, int H_kv,
                           int N, int d, float scale, int causal, void* fwd_workspace, size_t fwd_workspace_bytes,
                           void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Descriptor-based entry points: every option of the library in one problem
 * description, so that later options do not need new signatures.
 *   B, H, H_kv, N, d, scale, causal : as in fa_fwd_gqa / fa_bwd_gqa (H_kv = H for plain
 *                                     multi-head attention).
 *   window_left, window_right        : sliding-window (local) attention: query i sees key
 *                                     j only if i - window_left <= j <= i + window_right;
 *                                     -1 = unbounded on that side (both -1: no window).
 *                                     Combined with the causal mask (which already
 *                                     bounds the right side).  Every row keeps at least
 *                                     its own key.  ("Flash Attention uitgelegd: een
 *                                     uitgebreide gids" names sliding window attention for
 *                                     long contexts; the (left, right) convention is the
 *                                     reading taken.)  Values < -1 are FA_ERR_INVALID_ARG.
 * fa_attn_fwd needs a workspace (fa_attn_fwd_workspace_size bytes; the forward of
 * fa_fwd_ws); fa_attn_bwd as fa_bwd_gqa with fa_attn_bwd_workspace_size bytes.  The
 * backward must be given the same problem (window included) as the forward whose O, LSE
 * and residual it receives.  The workspace-size functions return 0 for an empty or
 * invalid problem (or a NULL descriptor).
 */
typedef struct fa_attn_problem {
  int B, H, H_kv, N, d;
  float scale;
  int causal;
  int window_left, window_right;
} fa_attn_problem;
FA_API size_t fa_attn_fwd_workspace_size(const fa_attn_problem* problem);
FA_API fa_status fa_attn_fwd(const fa_attn_problem* problem, const void* q, const void* k, const void* v, void* o,
                             float* lse, void* o_resid, void* workspace, size_t workspace_bytes,
                             fa_stream_t stream);
FA_API size_t fa_attn_bwd_workspace_size(const fa_attn_problem* problem);
FA_API fa_status fa_attn_bwd(const fa_attn_problem* problem, const void* q, const void* k, const void* v,
                             const void* o, const void* o_resid, const void* dout, const float* lse, float* dq,
                             float* dk, float* dv, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_attn_fwd_fp8_workspace_size / fa_attn_fwd_fp8 -- forward pass on 8-bit inputs.
 * ("Flash Attention uitgelegd: een uitgebreide gids", section "Native FP8-precisie";
 * "FlashAttention (EL)", section "FlashAttention-3 (2024)": FlashAttention-3 runs the
 * attention products in FP8 on the tensor cores.  The pages give no format or scaling
 * scheme; the reading taken is E4M3 operands with one descale factor per tensor.)
 *   problem          : as for fa_attn_fwd (grouped heads, causal mask, sliding window);
 *                      d must be 128 or 64 (FA_ERR_UNSUPPORTED otherwise).
 *   q                : const E4M3 (B, H, N, d), 16-byte aligned; k, v: const E4M3
 *                      (B, H_kv, N, d), 16-byte aligned.  One byte per element in the
 *                      OCP FP8 E4M3 encoding (bias 7, no infinities, 0x7F / 0xFF NaN).
 *   q_descale, k_descale, v_descale : positive finite floats; the attention is computed
 *                      for the real-valued inputs q_descale * Q, k_descale * K and
 *                      v_descale * V (FA_ERR_INVALID_ARG otherwise).
 *   o                : bf16 (B, H, N, d), 16-byte aligned, written.
 *   lse              : fp32 (B, H, N) or NULL, natural-log LSE of the scaled scores.
 *   workspace        : device buffer of fa_attn_fwd_fp8_workspace_size(problem) bytes
 *                      (256), 256-byte aligned, caller-owned; contents on entry do not
 *                      matter; one call at a time per workspace.
 * Both products run on the tensor cores in 8 bits with fp32 accumulation (the E4M3
 * products themselves are exact in fp32), and P V takes the probabilities P
 * rounded to E4M3 (round to nearest even; P <= 2^8 because the running maximum is
 * allowed to lag the true one by less than 8 in base-2 exponent).  The row sum that
 * divides O uses P before that rounding, so an output row differs from the exact
 * attention of the dequantized inputs by at most about 2^-4 times the P-weighted mean
 * of |V| (plus an absolute 2^-10 per key whose P falls below E4M3's normal range); LSE
 * is as accurate as the bf16 forward's.  No residual is produced (the backward takes
 * bf16 inputs).  Asynchronous on `stream`.
 */
FA_API size_t fa_attn_fwd_fp8_workspace_size(const fa_attn_problem* problem);
FA_API fa_status fa_attn_fwd_fp8(const fa_attn_problem* problem, const void* q, const void* k, const void* v,
                                 float q_descale, float k_descale, float v_descale, void* o, float* lse,
                                 void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_noalloc -- the backward pass of fa_bwd for callers that cannot allocate
 * device memory.  (The pages describe no such entry point; it is a service of this
 * library.)  Some callers have no way to obtain a workspace at the moment they run
 * the backward pass: a plugin's enqueue callback inside an engine that owns all
 * device memory and forbids allocation there, or a latency-bound loop in which
 * cudaMalloc (which may synchronise the device) is not acceptable.  This entry
 * point takes the arguments of fa_bwd_gqa with H_kv = H, minus the workspace, and uses
 * instead a scratch array compiled into the library: a file-scope device array of
 * FA_BWD_NOALLOC_MAX_WORKSPACE bytes (64 MiB) that every GPU which loads the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or any
 * other allocating routine.
 *   - Problems whose fa_bwd_workspace_size() exceeds FA_BWD_NOALLOC_MAX_WORKSPACE are
 *     rejected with FA_ERR_UNSUPPORTED before anything is launched (e.g. B*H*N*d up
 *     to about 8 million elements fits).
 *   - The first call on a device looks up the array's device address on that device
 *     (cudaGetSymbolAddress) and caches it; make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array, which keeps whatever the last call
 *     left in it.  Nothing in it needs to start at zero (each call overwrites every
 *     byte it reads), but calls whose work overlaps on the GPU -- on different
 *     streams, or from different host threads -- race on the array: serialise them.
 * Results are identical to fa_bwd_gqa (H_kv = H) with a workspace of its own.
 */
#define FA_BWD_NOALLOC_MAX_WORKSPACE ((size_t)64 << 20)
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                                const void* dout, const float* lse, float* dq, float* dk, float* dv, int B, int H,
                                int N, int d, float scale, int causal, fa_stream_t stream);

/*
 * fa_last_device_status -- synchronises `stream`, then reports what the kernels of this
 * library on the current device recorded since the last call: FA_ERR_TIMEOUT (a bounded
 * wait gave up) or FA_ERR_RANGE (an input beyond the value range above); the word is
 * then cleared.  FA_ERR_CUDA if the CUDA context holds an error, FA_OK otherwise.
 * fa_device_status is the same function under its earlier name.
 */
FA_API fa_status fa_last_device_status(fa_stream_t stream);
FA_API fa_status fa_device_status(fa_stream_t stream);

/*
 * fa_bwd_set_phase_events -- profiling hook.  With `events` pointing to two
 * cudaEvent_t handles (created by the caller), every later fa_bwd call made from
 * the same host thread records events[0] on its stream right after the
 * preprocess kernel and events[1] right after the dK/dV kernel, so a caller that
 * records its own events before and after the call can time each of the three
 * backward kernels.  NULL turns the hook off.  The library keeps only the pointer.
 */
FA_API void fa_bwd_set_phase_events(void* const* events);

/*
 * fa_selftest_wait_timeout -- self-test of the failure path: enqueues a one-CTA kernel in
 * which one thread waits, through the library's bounded-wait helper, on a barrier that
 * nothing ever completes.  The wait gives up after its wall-time limit (2 s) and records a
 * timeout, so a following fa_last_device_status(stream) returns FA_ERR_TIMEOUT (and clears it);
 * the CUDA context stays usable.  Nothing faults, traps or hangs.  Returns FA_OK once
 * enqueued.
 */
FA_API fa_status fa_selftest_wait_timeout(fa_stream_t stream);

/*
 * fa_selftest_exp2 -- self-test of the exponential that the softmax kernels evaluate on the
 * FMA pipe for part of their probabilities (instead of the special-function unit): y[i] =
 * that function of x[i] for i < n.  x, y: device fp32 arrays, 4-byte aligned.  The function
 * is meant for the arguments the kernels produce, x in [-126, 8]: on [-125.99, 8] its
 * relative error is at most 7.5e-5; closer to -126 the results are fp32 denormals (relative
 * error up to 1.5e-4), and below -126 it returns about 2^-126 -- values that round to 0 in
 * fp16.  Asynchronous on `stream`.  (A service of this library for its own tests; the pages
 * describe no such function.)
 */
FA_API fa_status fa_selftest_exp2(const float* x, float* y, int n, fa_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_API const char* fa_status_str(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
