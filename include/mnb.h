/*
 * mnb.h -- C ABI of libmnb.so: the MatMulNBits operator (weight-only 4-bit
 * block-quantized matmul) on NVIDIA B200 (sm_100a).
 *
 * The operator, as the model cards that ship it describe it:
 *   "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", intro and "Conversion details":
 *     MatMulNBits, 4 bits, block_size=32, is_symmetric=False; the decoder is
 *     ~95% MatMul ops ("Compression vs original").
 *   "int4 STT weights for sherpa-onnx", "Why int4 rather than the usual int8":
 *     weight-only, in blocks, activations untouched.
 *   "qwen3-asr-0.6b-onnx-int4-merged", "Provenance": block_size=64.
 *   "Qwen3-ASR-0.6B -- ONNX for the browser", "Pick a variant": q4 (fp32
 *     float tensors) and q4f16 (fp16 float tensors).
 *
 * Definitions (standard asymmetric int4):
 *   w[n][k] = (q[n][k] - zp[n][b]) * scale[n][b],  b = k / bs,
 *   zp = 8 for every block when no zero-point tensor is given,
 *   Y[m][n] = sum_k X[m][k] * w[n][k]              (Y = X . dequant(W)^T).
 *
 * Layout (row-major, contiguous, element 0 first):
 *   packed  uint8 [N][K/2]: element 2j of a row in the LOW nibble of byte j,
 *           element 2j+1 in the high nibble (equivalently [N][K/bs][bs/2]).
 *   scales  fp32 or fp16 [N][K/bs].
 *   zp      uint8 [N][ceil((K/bs)/2)]: block b in byte b/2, low nibble when b
 *           is even; an odd count leaves the last high nibble 0.  NULL = no
 *           zero points (zp = 8).
 *   X       [M][K] and Y [M][N] in the activation dtype.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer allocated and owned by the
 *     caller, except the size outputs of mnb_packed_sizes (host pointers).
 *     The library allocates no device memory and keeps no pointer after the
 *     call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronizes.
 *   - Arguments are validated on the host first; a failed check returns a
 *     negative MNB_ERR_* code, launches nothing, and sets a thread-local
 *     message readable with mnb_last_error().
 *   - Pointers to packed weights, activations and outputs must be 16-byte
 *     aligned (MNB_ERR_ALIGN otherwise); scales and zero points need only
 *     their element alignment.
 *   - Inputs must be finite.  Inputs and outputs must not overlap.
 */
#ifndef MNB_H
#define MNB_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MNB_API __attribute__((visibility("default")))
#else
#define MNB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MNB_F32 = 0, MNB_F16 = 1 } mnb_dtype;

enum {
    MNB_OK = 0,
    MNB_ERR_INVALID_ARG = -1, /* NULL pointer, negative size, unknown dtype     */
    MNB_ERR_SHAPE = -2,       /* bs not 32/64, K % bs != 0, size too large      */
    MNB_ERR_ALIGN = -3,       /* a pointer is not aligned as documented         */
    MNB_ERR_UNSUPPORTED = -4, /* a valid request the library does not serve     */
    MNB_ERR_CUDA = -5,        /* a CUDA runtime call or launch failed           */
    MNB_ERR_TIMEOUT = -6      /* a device-side bounded wait gave up: returned by
                                 mnb_device_status, which reads the word the
                                 kernels set (kernel launches return before the
                                 wait happens) */
};

/* Flags for mnb_gemv / mnb_gemm. */
enum {
    /* Launch with programmatic dependent launch: the kernel may start while
     * the previous kernel on `stream` is still running, and reads its WEIGHTS
     * (packed, scales, zp) before waiting for that kernel to finish; it reads X
     * and writes Y only after the wait.  Pass it only when no kernel still in
     * flight on the stream writes this call's weights. */
    MNB_FLAG_PDL = 1
};

/* Message describing the last failed call on this host thread ("" if none). */
MNB_API const char *mnb_last_error(void);

/* Library version string. */
MNB_API const char *mnb_version(void);

/* Bytes of the packed tensors of one [N, K] weight.  Host-only, no CUDA call.
 * Pages: byte counts of "qwen3-asr-0.6b-onnx-int4-merged" ("Why": 962 MB ->
 * 340 MB) follow from this layout with fp32 scales and packed 4-bit zp.
 * Errors: MNB_ERR_INVALID_ARG (NULL output, N < 0, bad dtype),
 *         MNB_ERR_SHAPE (bs not 32/64, K <= 0 or K % bs != 0). */
MNB_API int mnb_packed_sizes(int64_t N, int64_t K, int bs, mnb_dtype scale_t, int has_zp,
                     size_t *packed_bytes, size_t *scale_bytes, size_t *zp_bytes);

/* Block-wise round-to-nearest quantization of fp32 W [N][K] into the packed
 * layout ("Mega-ASR -- INT4 ONNX", "Conversion details": block_size=32,
 * is_symmetric=False, bits=4; "Qwen3-ASR-0.6B -- ONNX for the browser": RTN).
 *   has_zp = 1: lo = min(0, min v), hi = max(0, max v), scale = (hi - lo)/15,
 *               zp = clamp(rint(-lo/scale), 0, 15),
 *               q = clamp(rint(v/scale + zp), 0, 15)  (IEEE divide, then add;
 *               rint rounds half to even); scale == 0 gives zp = q = 0.
 *   has_zp = 0: zp = 8 implied, scale = max|v| / 7, q = clamp(rint(v/scale) + 8,
 *               0, 15); scale == 0 gives q = 8.  zp may be NULL.
 *   scale_t = MNB_F16 stores fp16_rn of the fp32 scale (q uses the fp32 one).
 * Results are bit-identical to a scalar fp32 evaluation of these formulas.
 * Writes packed, scales and (has_zp) zp completely.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN (W or packed not
 *         16-byte aligned), MNB_ERR_CUDA. */
MNB_API int mnb_quantize_rtn(const float *W, int64_t N, int64_t K, int bs, int has_zp,
                     uint8_t *packed, void *scales, mnb_dtype scale_t, uint8_t *zp,
                     void *stream);

/* W_out[n][k] = (q - zp) * scale, rounded once to out_t (fp32 or fp16) from
 * the exact product.  zp NULL = 8.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_dequantize(const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                   const uint8_t *zp, int64_t N, int64_t K, int bs, void *W_out,
                   mnb_dtype out_t, void *stream);

/* Decode-shaped MatMulNBits, 1 <= M <= 16 with fp32 activations and
 * 1 <= M <= 32 with fp16 activations (the autoregressive step of
 * "Qwen3-ASR-0.6B -- ONNX for the browser", "Graph contracts": decoder_step,
 * input_embeds [1, 1, 1024], batched or over a few appended prompt tokens).
 * Y = X . dequant(W)^T.
 *   act_t  = dtype of X and Y (fp32 or fp16); scale_t = dtype of scales.
 *   Accumulation is fp32.  Bandwidth-bound: streams the packed weights once.
 *   With fp16 activations an fp32 scale takes part as fp16_rn(scale) (the
 *   fp16 arithmetic of the q4f16 graphs); with fp32 activations every step
 *   is fp32.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN,
 *         MNB_ERR_UNSUPPORTED (M above the limit), MNB_ERR_CUDA. */
MNB_API int mnb_gemv(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales,
             mnb_dtype scale_t, const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K,
             int bs, unsigned flags, void *stream);

/* Gate and up projections of the decoder's SwiGLU MLP with its activation fused
 * in ("Qwen3-ASR-1.7B ONNX", "Architecture": Qwen3 decoder with SwiGLU):
 *   Y[m][i] = silu(G[m][i]) * U[m][i],  G = X . dequant(Wg)^T, U = X . dequant(Wu)^T,
 *   silu(x) = x / (1 + exp(-x)), from the fp32 sums, rounded once to fp16.
 * The weight [N][K] holds the gate and up rows interleaved in groups of 16 rows:
 * rows 16j .. 16j+7 are gate rows 8j .. 8j+7, rows 16j+8 .. 16j+15 the up rows
 * of the same outputs (scales and zero points follow their rows).  Y is
 * [M][N/2].  fp16 activations, 1 <= M <= 16, N % 16 == 0.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN,
 *         MNB_ERR_UNSUPPORTED (M > 16), MNB_ERR_CUDA. */
MNB_API int mnb_gemv_swiglu(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                    const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, unsigned flags,
                    void *stream);

/* The output projection of a decode step fused with greedy decoding
 * ("Qwen3-ASR-0.6B -- ONNX for the browser", "Building the prompt" step 5:
 * greedy decode with decoder_step, logits [1, 1, 151936]).  Computes Y exactly
 * as mnb_gemv (fp16 activations) and, for every token m,
 *   ids[m]     = the smallest n with Y[m][n] = max_n' Y[m][n']  (the fp16 values
 *                written to Y; the first maximum on ties),
 *   max_out[m] = that maximum as fp32 (max_out may be NULL).
 *   1 <= M <= 16, N >= 1.  ids (int32 [M]) and max_out are device pointers.
 *   workspace: device buffer of at least mnb_gemv_argmax_workspace_bytes(M)
 *   bytes (for the current device), 16-byte aligned, ZERO-FILLED before its
 *   first use.  Its first bytes count the CTAs that finished; the last one
 *   sets the count back to zero, so a workspace stays usable across calls; the
 *   rest is scratch.  Calls that share a workspace must not run concurrently
 *   on the GPU.
 * Errors: MNB_ERR_INVALID_ARG (also: workspace too small), MNB_ERR_SHAPE,
 *         MNB_ERR_ALIGN, MNB_ERR_UNSUPPORTED (M outside [1, 16]), MNB_ERR_CUDA. */
MNB_API size_t mnb_gemv_argmax_workspace_bytes(int64_t M);   /* 0 when M is outside [1, 16] */
MNB_API int mnb_gemv_argmax(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                    const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, int32_t *ids,
                    float *max_out, void *workspace, size_t ws_bytes, unsigned flags, void *stream);

/* mnb_gemv_argmax without a workspace argument.  No counterpart on the pages:
 * it is for callers that cannot hand this library device memory -- a plug-in
 * whose host application owns every device allocation through its own pool,
 * or a decode loop on a latency-critical thread that must not call the device
 * allocator (which can block, or fail for lack of memory, between two tokens).
 * Same arguments and results as mnb_gemv_argmax, minus workspace/ws_bytes.
 * The scratch is a device array inside libmnb.so: 64 KiB on every GPU that
 * loads the library, held until the process exits.  With 148 SMs that covers
 * every M in [1, 16]; a request needing more returns MNB_ERR_SHAPE with a
 * message.  Nothing is allocated: the first call on each device looks up the
 * array's device address (make that first call before any stream capture)
 * and keeps it for the life of the process, so a cudaDeviceReset of that
 * device makes later calls unusable (the kept address is stale); each call
 * clears the array's counter on `stream` before its kernel.
 * All calls on one GPU share the one array, which keeps the last call's
 * contents: calls that may run at the same time on the GPU (other streams,
 * other host threads) race on it and must be serialized by the caller.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN,
 *         MNB_ERR_UNSUPPORTED (M outside [1, 16]), MNB_ERR_CUDA. */
MNB_API int mnb_gemv_argmax_noalloc(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                            const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs,
                            int32_t *ids, float *max_out, unsigned flags, void *stream);

/* Prefill-shaped MatMulNBits on the tensor cores, any M >= 1 (tuned for
 * M >= 64: the full-length prefill of "Mega-ASR -- INT4 ONNX", "What's in this
 * repo": decoder_prefill).  Y = X . dequant(W)^T with fp16 X, scales and Y (the
 * q4f16 variant of "Qwen3-ASR-0.6B -- ONNX for the browser", "Pick a
 * variant"); each weight is dequantized to fp16_rn((q - zp) * scale), the
 * value mnb_dequantize writes, and the products are accumulated in fp32.
 *   act_t and scale_t must be MNB_F16; N must be a multiple of 128 and K of 64.
 * One CTA per (128-row tile, token tile); when those leave SMs idle, K is
 * split over a thread-block cluster whose ranks add their partial sums in
 * rank order through distributed shared memory, so results are the same, bit
 * for bit, on every call.
 * A device-side wait that exceeds its iteration limit makes the kernel stop,
 * sets a bit in the library's device status word (see mnb_device_status) and
 * leaves Y incomplete; the call itself returned MNB_OK by then.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN,
 *         MNB_ERR_UNSUPPORTED (fp32 activations or fp32 scales), MNB_ERR_CUDA. */
MNB_API int mnb_gemm(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales,
             mnb_dtype scale_t, const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K,
             int bs, unsigned flags, void *stream);

/* The MatMulNBits operator for any number of tokens: the same
 * Y = X . dequant(W)^T (layouts, tolerances and errors as mnb_gemv/mnb_gemm)
 * on the kernel that serves M best.  Decode ("Graph contracts":
 * decoder_step), prefill of a prompt appended to a cached one (a few to a few
 * dozen new tokens) and full prefill (decoder_init / decoder_prefill) all take
 * this one call:
 *   M <= 24 with fp16 X (M <= 16 with fp32 X): one mnb_gemv (measured faster
 *     than the tensor-core GEMM up to 24 tokens);
 *   M >= 25 with fp16 X and scales, N % 128 == 0, K % 64 == 0: mnb_gemm;
 *   otherwise (fp32 X or scales, or shapes the GEMM does not take):
 *     mnb_gemv launches of up to 24 (fp16 X) or 16 (fp32 X) tokens.
 * Requires X, packed and Y 16-byte aligned.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_matmul(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                       const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, unsigned flags,
                       void *stream);

/* int8 embedding lookup ("Qwen3-ASR-0.6B -- ONNX for the browser",
 * "Building the prompt" step 4 and "Pick a variant": embed_tokens.int8.bin +
 * embed_scales.f32.bin):
 *   out[t][d] = round_out_t( fp32(table[ids[t]][d]) * row_scales[ids[t]] ),
 * the product taken in fp32 and rounded once more to fp16 when out_t is fp16.
 *   table int8 [V][D], row_scales fp32 [V], ids int32 [T], out [T][D].
 * An id outside [0, V) yields a zero row and, when status != NULL, sets bit 0
 * of the device int *status (atomic OR; the caller clears it).  Never traps.
 * Requires D % 16 == 0 and 16-byte aligned table and out.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_embed_gather(const int8_t *table, const float *row_scales, int64_t V, int64_t D,
                     const int32_t *ids, int64_t T, void *out, mnb_dtype out_t, int *status,
                     void *stream);

/* ---- a whole decode step in one launch ----------------------------------
 * The decoder step of "Qwen3-ASR-0.6B -- ONNX for the browser" ("Graph
 * contracts": decoder_step) and of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)"
 * is a sequence of MatMulNBits calls, 28 layers x 7 projections plus the
 * lm_head, each small enough that a launch per call costs more than its
 * weight traffic.  mnb_gemv_chain runs such a sequence ("tasks") as one
 * persistent kernel: per task the same Y = X . dequant(W)^T as mnb_gemv with
 * fp16 activations, fp16 scales and fp32 accumulation.
 *
 * Task j with wait != 0 reads its X only after tasks 0..j-1 have completed,
 * so X may be (part of) an earlier task's Y; with wait == 0 its X must not be
 * written by any task of the chain.  Task 0's X is read after the stream's
 * earlier work (and, with MNB_FLAG_PDL, after the previous kernel completes).
 * Tasks may share X; Y buffers must not overlap any task's X, W or another Y.
 *
 * Two steps.  mnb_gemv_chain_plan (host only, no device work) checks every
 * task, encodes its tensor map and writes a plan of
 * mnb_gemv_chain_plan_bytes(ntasks) bytes into caller memory.  The caller
 * copies those bytes unchanged to device memory (64-byte aligned) and calls
 * mnb_gemv_chain with both copies: the host copy for the launch shape, the
 * device copy for the kernel.  A plan holds device addresses and is valid for
 * the device that was current when it was made, for as long as every buffer
 * it names stays allocated; the same plan may be launched any number of
 * times (and captured in a CUDA graph).
 *
 * Requirements per task: N % 16 == 0, K % 256 == 0 (K % 512 == 0 for block
 * 64 with zero points); X and packed 16-byte aligned; scales 16-byte (block
 * 32) or 8-byte (block 64) aligned; zp 4-byte aligned; Y 2-byte aligned.
 * All tasks share M (1..8), the block size and the presence of zero points.
 *
 * workspace: mnb_gemv_chain_workspace_bytes(ntasks) bytes of device memory,
 * zero-filled before the first call; every call that completes leaves it
 * zero-filled again.  Calls sharing a workspace must be stream-ordered.
 * Failure: a wait inside the kernel that exceeds 2 s sets bit 1 (a weight
 * copy) or bit 2 (a task's inputs) of the status word read by
 * mnb_device_status; the kernel then exits early, Y is undefined and the
 * workspace must be zero-filled again.  A call that finds the workspace's
 * abort word still set (a failed call before it) runs no task, writes no Y
 * and sets bit 3.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN,
 *         MNB_ERR_UNSUPPORTED (M > 8, mixed layouts), MNB_ERR_CUDA. */
typedef struct mnb_gemv_task {
    const void *X;          /* fp16 [M][K] */
    const uint8_t *packed;  /* [N][K/2] */
    const void *scales;     /* fp16 [N][K/bs] */
    const uint8_t *zp;      /* [N][ceil(K/bs/2)] or NULL (zero point 8) */
    void *Y;                /* fp16 [M][N] */
    int64_t N, K;
    int32_t wait;           /* != 0: X is read after tasks 0..j-1 complete */
    int32_t reserved;       /* 0 */
} mnb_gemv_task;

MNB_API size_t mnb_gemv_chain_plan_bytes(int ntasks);        /* 0 when ntasks is outside [1, 65536] */
MNB_API size_t mnb_gemv_chain_workspace_bytes(int ntasks);   /* 0 when ntasks is outside [1, 65536] */
MNB_API int mnb_gemv_chain_plan(const mnb_gemv_task *tasks, int ntasks, int64_t M, int bs, void *plan,
                                size_t plan_bytes);
MNB_API int mnb_gemv_chain(const void *plan, const void *plan_device, void *workspace, size_t ws_bytes,
                           unsigned flags, void *stream);

/* ---- GPTQ quantization into the packed layout -----------------------------
 * "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", "Conversion details" (algo=GPTQ,
 * block_size=32, is_symmetric=False, bits=4) and "GPTQ calibration" (the
 * Hessian accumulated from calibration activations, a Cholesky factorisation
 * of its inverse, the inner loop in fp32 on the GPU, a diagonal-jitter retry
 * when the fp32 factorisation fails).  The algorithm is the published GPTQ;
 * the three calls below are its three stages.  Their outputs feed every
 * MatMulNBits entry point above unchanged. */

/* H (+)= X^T X: H fp32 [K][K] (row-major, full), X [T][K] fp32 or fp16
 * calibration inputs (the activations the weight meets).  accumulate = 0
 * overwrites H, 1 adds to it (several calibration batches).  The usual 2/T
 * factor is left out: no result of the method depends on it.  fp32
 * accumulation.  1 <= K <= 8192.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_gptq_hessian(const void *X, mnb_dtype x_t, int64_t T, int64_t K, float *H, int accumulate,
                             void *stream);

/* Bytes of the workspace of mnb_gptq_prepare (0 when K is outside [1, 8192]). */
MNB_API size_t mnb_gptq_workspace_bytes(int64_t K);

/* From H (read only): dead[k] = 1 where H_kk == 0 (a feature the calibration
 * never activated: its diagonal becomes 1 and mnb_gptq_quantize zeroes its
 * weights), the diagonal damped by percdamp x its mean (0.01 is usual), and
 * U fp32 [K][K] = the upper Cholesky factor of the damped H^-1 (H^-1 = U^T U,
 * zeros below the diagonal).  If the fp32 factorisation meets a non-positive
 * pivot it starts again with 10x the damping (0.001 after percdamp = 0), up
 * to three times; *damp_used
 * (host pointer, may be NULL) receives the damping that succeeded.  HOST-
 * BLOCKING: synchronizes `stream` once per attempt.  workspace: device memory
 * of mnb_gptq_workspace_bytes(K) bytes, 16-byte aligned, any contents.
 * Errors: MNB_ERR_INVALID_ARG (also: no attempt succeeded), MNB_ERR_SHAPE,
 *         MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_gptq_prepare(const float *H, int64_t K, float percdamp, float *U, uint8_t *dead, void *workspace,
                             size_t ws_bytes, float *damp_used, void *stream);

/* GPTQ of fp32 W [N][K] (read only) with U from mnb_gptq_prepare and its dead
 * flags (dead may be NULL: none).  Per row, column by column: a block's scale
 * and zero point come from the row's current values of the block (the RTN
 * rule of mnb_quantize_rtn, same has_zp variants), the code is the RTN code,
 * and the rounding error err = (w_i - (q_i - zp) * scale) / U_ii is fed back:
 * w_k -= err * U_ik for k > i.  Every step is one fp32 operation in that
 * order, so the codes do not depend on the launch shape.  Writes packed,
 * scales (fp16_rn of the fp32 scale when scale_t is MNB_F16) and zp in the
 * layout above.  K <= 8192, K % bs == 0.
 * Errors: MNB_ERR_INVALID_ARG, MNB_ERR_SHAPE, MNB_ERR_ALIGN, MNB_ERR_CUDA. */
MNB_API int mnb_gptq_quantize(const float *W, const float *U, const uint8_t *dead, int64_t N, int64_t K, int bs,
                              int has_zp, uint8_t *packed, void *scales, mnb_dtype scale_t, uint8_t *zp,
                              void *stream);

/* Reads (and, if clear != 0, zeroes) the library's device status word on the
 * current device into *status_out: bit 0 = a GEMM or GEMV mbarrier wait timed
 * out; bits 1-3 = mnb_gemv_chain (see there).  Synchronizes the device.
 * Returns MNB_ERR_TIMEOUT (with *status_out written) when any of bits 0-2 is
 * set, i.e. a bounded wait inside a kernel gave up since the word was last
 * cleared; MNB_OK otherwise.
 * Errors: MNB_ERR_INVALID_ARG (NULL), MNB_ERR_CUDA, MNB_ERR_TIMEOUT. */
MNB_API int mnb_device_status(unsigned *status_out, int clear);

#ifdef __cplusplus
}
#endif

#endif /* MNB_H */
