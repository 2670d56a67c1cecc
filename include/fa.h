/*
 * fa.h -- C ABI of the exact-attention library for NVIDIA B200 (sm_100a).
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T [+ mask]) V
 *
 * (the formula of FlashAttention (DE), section "Problematik der Standard-Attention"), as one
 * fused, tiled forward kernel that never writes the N x N score matrix to device memory
 * (FlashAttention (DE), sections "Tiling und blockweise Verarbeitung", "Online-Softmax-
 * Berechnung" and "Zusammenfassen von Operationen in einem CUDA-Kernel"), and a backward pass
 * that keeps only the per-row log-sum-exp and recomputes the probabilities block by block
 * (flash-attention glossary page, "Hoe werkt het?", item "Herberekening").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.     Q, K, V, O, dO, dQ, dK, dV are bf16, contiguous, shape [B, H, N, d]
 *             (row-major: d fastest, then N, then H, then B).  lse is fp32 [B, H, N].
 * Sizes.      B >= 1, H >= 1, 1 <= N, d in {64, 128, 256} (FlashAttention (DE),
 *             "FlashAttention-2 (2023)": heads of size 256; fa_bwd_noalloc takes 64 and 128
 *             only); B*H*N*d must fit in 2^31 elements.
 * Mask.       causal != 0 hides key j from query i when j > i (top-left alignment, N queries
 *             and N keys).  seqlens, when not NULL, is a DEVICE int32 array of B key lengths
 *             L_b with 1 <= L_b <= N: keys j >= L_b of batch b are hidden from every query.
 *             Both masks combine by AND.  Query rows i >= L_b are still computed (they attend
 *             to the visible keys).  A length outside [1, N] is reported through the device
 *             error flag as FA_ERR_INVALID_ARG and treated as clamped to [1, N].
 * scale.      Multiplies Q K^T; must be finite and > 0 (1/sqrt(d) is the usual choice).
 * Pointers.   Device pointers, 16-byte aligned, not aliasing one another (outputs never alias
 *             inputs).  The caller allocates and owns every buffer, including the workspace.
 * Streams.    `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call only
 *             validates its arguments and enqueues kernels on `stream`; FA_OK means
 *             "validated and launched".  Errors found on the device (a bad length, a wait
 *             that timed out) are recorded in a per-device error flag that
 *             fa_check_device_error() reads.
 * Errors.     No exception crosses the ABI.  A rejected call launches nothing and leaves every
 *             output untouched.
 * Device.     Requires a compute capability 10.0 GPU (B200); otherwise FA_ERR_UNSUPPORTED.
 * Threads.    Calls may come from several host threads; calls on one stream run in order.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

/* Same type as cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* a NULL/misaligned pointer, a size or scale out of range      */
    FA_ERR_UNSUPPORTED = 2,  /* head dim not 64/128/256 for this entry point, or not an sm_100 GPU */
    FA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, tensor map, ...)  */
    FA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (reported by the flag)   */
    FA_ERR_WORKSPACE = 5     /* fa_bwd: workspace NULL, misaligned or smaller than required */
} fa_status;

/*
 * Forward pass.
 *   q, k, v   in : bf16 [B, H, N, d]
 *   o         out: bf16 [B, H, N, d]   O = softmax(scale * Q K^T + mask) V
 *   lse       out: fp32 [B, H, N]      lse_i = ln sum_{j visible} exp(scale * q_i . k_j),
 *                                      the "normalisation values" the backward pass keeps
 *                                      (flash-attention glossary page, "Herberekening").
 * One fused kernel: Q/K/V tiles staged through shared memory by TMA, Q K^T and P V on the
 * tensor cores (tcgen05, accumulators in tensor memory), online softmax with a running row
 * maximum and row sum (FlashAttention (DE), "Online-Softmax-Berechnung").  Allocates nothing.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, float scale, int causal, const int* seqlens,
                 fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes (0 if the sizes are invalid).
 * The workspace holds D = rowsum(dO * O) and |dO_i| (fp32 [B, H, N] each), per-128-row-chunk
 * maxima of |v_j| and |k_jl| (fp32 [B, H, N_pad / 128, 2]) and the int32 fixed-point dQ
 * accumulator ([B, H, N_pad, d]), N_pad = N rounded up to 128.  Its contents need not be
 * initialised; fa_bwd writes everything it reads.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass (training).  Recomputes P block by block from lse (flash-attention glossary
 * page, "Herberekening") and forms the ordinary derivative of the forward formula:
 *     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
 *     dK = scale * dS^T Q,  dQ = scale * dS K.
 *   q, k, v, o, dO in : bf16 [B, H, N, d]; o is the forward output for the same inputs
 *   lse            in : fp32 [B, H, N] from fa_fwd with the same inputs and mask
 *   dq, dk, dv     out: bf16 [B, H, N, d], fully overwritten
 *   workspace      scratch of at least fa_bwd_workspace_size(B, H, N, d) bytes, 16-byte
 *                  aligned, owned by the caller, not used concurrently by another call.
 * The dQ sum over key blocks is exact integer (fixed-point) arithmetic: each key block's
 * contribution to query row i is rounded once to 2^-29 of an a-priori bound of row i
 * (2 |dO_i| max_j |v_j| max |k|) and the integer sum does not depend on the order in which
 * key blocks arrive, so repeated calls on the same inputs give bitwise identical dq, dk, dv.
 * Inputs so large that this bound is not finite in fp32 (norms beyond 3.4e38) leave that
 * row's dq at 0 and record FA_ERR_INVALID_ARG in the device error flag.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 int B, int H, int N, int d, float scale, int causal, const int* seqlens,
                 void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_selftest_wait_timeout -- a check of the failure path: launches a one-CTA kernel whose
 * only work is a bounded wait (the same mbarrier wait every kernel of this library uses) on a
 * barrier that nothing ever completes.  The wait gives up after the current limit
 * (fa_set_wait_timeout_ns, at least 1 ms) and records FA_ERR_TIMEOUT in the device error flag,
 * which the next fa_check_device_error returns; the context stays usable.  Nothing faults,
 * traps or hangs.  Returns FA_OK when launched.
 */
FA_API fa_status fa_selftest_wait_timeout(fa_stream_t stream);

/*
 * Index checks.  The library also comes as a checking build (libfa_debug.so, the same sources
 * compiled with FA_DEBUG), a stand-in for a memory sanitizer: in it every plain load and store
 * of global memory in the kernels (the accesses not made by TMA, whose tensor maps bound them)
 * first checks its index against the buffer it belongs to; an index outside records
 * FA_ERR_INVALID_ARG in the device error flag and the access is skipped.  Nothing traps.
 * fa_debug_checks returns 1 in that build and 0 in the release build.
 *
 * fa_selftest_bounds exercises that check: one thread stores `value` to buf[n - 1] and to
 * buf[n] (one past a caller-owned device buffer of n >= 1 ints, 4-byte aligned) through it, so
 * buf[n - 1] is written, buf[n] is not, and the next fa_check_device_error returns
 * FA_ERR_INVALID_ARG.  The release build returns FA_ERR_UNSUPPORTED and launches nothing.
 */
FA_API int fa_debug_checks(void);
FA_API fa_status fa_selftest_bounds(int* buf, int n, int value, fa_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the calling device's error flag.
 * Returns FA_OK, FA_ERR_INVALID_ARG (a sequence length outside [1, N] was seen, or a
 * backward row whose fixed-point bound overflowed fp32),
 * FA_ERR_TIMEOUT (a device-side wait gave up; the outputs of that call are undefined) or
 * FA_ERR_CUDA (the synchronisation itself failed).
 */
FA_API fa_status fa_check_device_error(fa_stream_t stream);

/*
 * Upper bound, in nanoseconds, on every wait inside the kernels (pipeline barriers and the
 * ordered dQ reduction).  When a wait exceeds it, the kernel records FA_ERR_TIMEOUT, stops
 * its work and exits instead of hanging.  Default 4e9 (4 s); values below 1e6 are raised to
 * 1e6.  Applies to launches made after the call, on every device.
 */
FA_API void fa_set_wait_timeout_ns(uint64_t ns);

/*
 * Measurement hook.  The next attention call made on this host thread (any fa_fwd*, fa_bwd*,
 * fa_fwd_fp8 or fa_fwd_decode) records `start_event` on its stream immediately before its main
 * fused kernel and `stop_event` immediately after it (the backward's preprocess and dQ
 * convert kernels, and the decode combine kernel, fall outside), then forgets both.  The
 * events are cudaEvent_t handles the caller created (NULL: not recorded).  This lets a caller
 * time one kernel with CUDA events on the launching stream.
 */
FA_API void fa_set_kernel_timing_events(void* start_event, void* stop_event);

/*
 * Grouped-query / multi-query attention (FlashAttention (DE), section on FlashAttention-2:
 * support for multi-query attention).  Same as fa_fwd / fa_bwd, except that K and V (and dK,
 * dV) have H_kv heads, [B, H_kv, N, d], with H % H_kv == 0: query head h attends with key/value
 * head h / (H / H_kv) (consecutive query heads share one key/value head; H_kv = 1 is
 * multi-query attention, H_kv = H is fa_fwd / fa_bwd).  dK and dV of a key/value head are the
 * sums over its query heads, formed inside one CTA in a fixed order (no atomics), so repeated
 * calls stay bitwise identical.  The workspace is fa_bwd_workspace_size(B, H, N, d) (query
 * heads).  H_kv outside [1, H] or not dividing H: FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int H_kv, int N, int d, float scale, int causal,
                            const int* seqlens, fa_stream_t stream);
FA_API fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                            const void* dO, const float* lse, void* dq, void* dk, void* dv,
                            int B, int H, int H_kv, int N, int d, float scale, int causal,
                            const int* seqlens, void* workspace, size_t workspace_bytes,
                            fa_stream_t stream);

/*
 * Packed variable-length sequences.  The pages print no packed layout; they speak of batches
 * whose sequences differ in length (the padded BERT workload of FlashAttention (DE),
 * "Empirische Ergebnisse").  This is the same computation with the sequences stored back to
 * back instead of padded to a common length, so that no padding row is read or written.
 * Sequence b is rows [cu_seqlens[b], cu_seqlens[b+1]) of
 *   q, o, dO, dq   bf16 [total, H, d]      (row t, head h at (t * H + h) * d)
 *   k, v, dk, dv   bf16 [total, H_kv, d]
 *   lse            fp32 [H, total]          (natural-log units, as in fa_fwd)
 * and is an independent attention problem: its queries attend to its own keys only (and, when
 * causal, to keys j <= i of the same sequence, counted from the sequence's first row).  H_kv
 * follows fa_fwd_gqa.  Rows of `o`, `lse`, `dq`, `dk`, `dv` outside every sequence
 * ([cu_seqlens[B], total)) are not written.
 *   cu_seqlens   device int32 [B + 1], 4-byte aligned, non-decreasing, cu_seqlens[0] >= 0,
 *                cu_seqlens[B] <= total; empty sequences are allowed.
 *   max_seqlen   >= the longest sequence (it sizes the grid and the backward workspace:
 *                fa_bwd_workspace_size(B, H, max_seqlen, d)).
 * A sequence that breaks these rules (found on the device) is skipped and FA_ERR_INVALID_ARG
 * is recorded for fa_check_device_error.  Host-side checks as in fa_fwd, plus total >= 1 and
 * total * H * d < 2^31.  The padded accumulators of the backward workspace keep the
 * [B, H, max_seqlen] shape.
 */
FA_API fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens, int B, int max_seqlen, int total, int H,
                               int H_kv, int d, float scale, int causal, fa_stream_t stream);
FA_API fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                               const void* dO, const float* lse, void* dq, void* dk, void* dv,
                               const int* cu_seqlens, int B, int max_seqlen, int total, int H,
                               int H_kv, int d, float scale, int causal, void* workspace,
                               size_t workspace_bytes, fa_stream_t stream);

/*
 * Decode: a few new queries per sequence against a long key/value cache (token-by-token
 * generation; FlashAttention (DE), "Spezialisierte Lösungen": FlashInfer's processing of the
 * KV cache in streaming generation, FlashDecoding).  Forward only.
 *   q, o           bf16 [B, H, Nq, d]        Nq >= 1 new queries per sequence
 *   k_cache, v_cache bf16 [B, H_kv, N, d]    N = cache capacity; H % H_kv == 0 and query head h
 *                                            reads cache head h / (H / H_kv)
 *   lse            fp32 [B, H, Nq]           natural-log units
 *   cache_lens     device int32 [B] valid cache rows L_b in [1, N] (rows >= L_b are ignored),
 *                  or NULL for L_b = N; out-of-range values are clamped and reported.
 *   causal         query i (0-based of Nq) is position L_b - Nq + i and sees keys
 *                  j <= L_b - Nq + i (aligned to the end of the cache); a query that sees no
 *                  key gets O = 0 and lse = -inf.
 *   splits         key ranges per (sequence, cache head) computed by separate CTAs and merged
 *                  by their log-sum-exp; 0 = fa_decode_num_splits(..., cache_lens != NULL).  Ranges hold whole key
 *                  blocks (64 keys for d <= 128, 128 for d = 256), so the count used may be
 *                  lower than the one requested.
 *   workspace      device, 16-byte aligned, >= fa_decode_workspace_size(B, H, Nq, d, splits)
 *                  bytes for the requested splits when they exceed 1; may be NULL otherwise.
 * d in {64, 128, 256}.  The result is exact for every `splits` (up to rounding: different
 * splits round differently; the same splits give identical bits).
 */
/* Automatic split count; ragged != 0 when per-sequence cache lengths will be passed (more
 * ranges, so that the longest sequences do not dominate). */
FA_API int fa_decode_num_splits(int B, int H, int H_kv, int Nq, int N, int d, int ragged);
FA_API size_t fa_decode_workspace_size(int B, int H, int Nq, int d, int splits);
FA_API fa_status fa_fwd_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                               float* lse, const int* cache_lens, int B, int H, int H_kv,
                               int Nq, int N, int d, float scale, int causal, int splits,
                               void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * FP8 forward (FlashAttention-3's FP8 mode; Russian article, "FlashAttention-3 (2024)").
 * q, k, v hold OCP FP8 E4M3 codes ("fn" variant, one byte each), layout as fa_fwd_gqa with
 * d = 128 only: q [B, H, N, 128], k, v [B, H_kv, N, 128].  The values they stand for are
 * code * descale with per-(batch, head) fp32 factors q_descale [B, H], k_descale [B, H_kv],
 * v_descale [B, H_kv] (device arrays, 4-byte aligned; NULL means 1).  O (bf16 [B, H, N, 128])
 * and lse (fp32 [B, H, N]) are those of exact attention of the dequantised values, up to the
 * rounding of the probabilities to e4m3 before the P V product: |O - O_exact| is bounded per
 * element by 2^-4 * sum_j P_ij |v_jc| + 2^-14 * sum_{visible j} |v_jc| (relative e4m3 rounding,
 * and absolute underflow of probabilities below 2^-14 of the row's largest) plus bf16 output
 * rounding.  Masks, seqlens and errors as fa_fwd.  d != 128: FA_ERR_UNSUPPORTED.
 */
FA_API fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                            const float* k_descale, const float* v_descale, void* o, float* lse,
                            int B, int H, int H_kv, int N, int d, float scale, int causal,
                            const int* seqlens, fa_stream_t stream);

/*
 * fa_bwd_noalloc -- the backward pass without any device allocation.  The pages have no
 * counterpart of this entry point; it exists for callers that cannot allocate device memory:
 * a process that reserves its whole device-memory budget for its own pool up front, or a
 * latency-critical loop that must not call cudaMalloc / cudaFree (they can block and
 * synchronise the device).
 *
 * It computes exactly what fa_bwd computes, with the same kernels, arguments, layouts and
 * results, but its scratch (the workspace fa_bwd takes from the caller) is a fixed area of
 * FA_BWD_NOALLOC_SCRATCH_BYTES inside this library's own device code image: every GPU on which
 * that image is loaded holds the area until the process exits.  The caller still provides
 * every input and output buffer.
 *   error_flag  optional caller-owned device int (4-byte aligned): device-side errors of this
 *               call (a bad sequence length, a wait that timed out) are stored there as an
 *               fa_status code; it is never cleared by the library.  NULL: not reported.
 * Limits and rules:
 *   - Problems whose fa_bwd_workspace_size(B, H, N, d) exceeds FA_BWD_NOALLOC_SCRATCH_BYTES
 *     are rejected with FA_ERR_WORKSPACE (e.g. B*H = 31, N = 4096, d = 128 fits;
 *     B*H = 32 at the same N and d does not).
 *   - All calls on a device share the one scratch area and each call overwrites it.  Calls
 *     whose kernels overlap on the GPU (other streams, other host threads) race and give
 *     wrong results: issue them on one stream, or order them yourself.
 *   - The first call on a device performs a one-time set-up on the host (it looks up the
 *     scratch area's device address); make that first call before any stream capture.
 *   - When the area is placed in device memory depends on CUDA's module loading.  Under lazy
 *     loading (the default since CUDA 12.2) it is placed by that first call on each device,
 *     not when the library is loaded: a caller that reserves the rest of the device memory for
 *     its own pool should make the first call before reserving it (or run with
 *     CUDA_MODULE_LOADING=EAGER, which places the area when the library's code is loaded).  If
 *     the first call finds no room for the area it returns FA_ERR_WORKSPACE and launches
 *     nothing; a later call tries again.
 *   - No cudaMalloc, cudaFree or other allocating call is made by this entry point.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                int B, int H, int N, int d, float scale, int causal,
                                const int* seqlens, int* error_flag, fa_stream_t stream);

/* Static, human-readable name of a status code. */
FA_API const char* fa_status_string(fa_status s);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
