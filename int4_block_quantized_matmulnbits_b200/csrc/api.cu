// api.cu -- the extern "C" entry points of libmnb: host-side argument checks,
// then the launchers of the kernel files.  Nothing here touches the device
// before every check has passed.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace mnb {

static thread_local char g_msg[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return code;
}

void clear_error() { g_msg[0] = 0; }

int check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MNB_OK;
}

EncodeTiledFn tensor_map_encoder() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

int device_sm_count() {
    static int counts[128] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128)
        return 148;
    if (counts[dev] <= 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

cudaError_t ensure_dynamic_smem(const void *kernel, int bytes, int *cache) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (bytes <= cache[dev])
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        cache[dev] = bytes;   // two threads racing here both set the same attribute
    return e;
}

// Limits: sizes fit comfortably in 32-bit element indices of one row and in
// 64-bit byte offsets overall.
static const int64_t kMaxDim = (int64_t)1 << 30;

static int check_weight_shape(const char *fn, int64_t N, int64_t K, int bs) {
    if (N < 0 || K < 0)
        return fail(MNB_ERR_INVALID_ARG, "%s: negative size (N=%lld K=%lld)", fn, (long long)N,
                    (long long)K);
    if (bs != 32 && bs != 64)
        return fail(MNB_ERR_SHAPE, "%s: block size %d not in {32, 64}", fn, bs);
    if (K == 0 || K % bs != 0)
        return fail(MNB_ERR_SHAPE, "%s: K=%lld is not a positive multiple of bs=%d", fn,
                    (long long)K, bs);
    if (N > kMaxDim || K > kMaxDim)
        return fail(MNB_ERR_SHAPE, "%s: N or K above 2^30", fn);
    return MNB_OK;
}

static int check_dtype(const char *fn, const char *what, int t) {
    if (t != MNB_F32 && t != MNB_F16)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown %s dtype %d", fn, what, t);
    return MNB_OK;
}

static int check_matmul_args(const char *fn, const void *X, int act_t, const uint8_t *packed,
                             const void *scales, int scale_t, void *Y, int64_t M, int64_t N,
                             int64_t K, int bs) {
    int rc;
    if ((rc = check_dtype(fn, "activation", act_t)) || (rc = check_dtype(fn, "scale", scale_t)))
        return rc;
    if ((rc = check_weight_shape(fn, N, K, bs)))
        return rc;
    if (M < 0)
        return fail(MNB_ERR_INVALID_ARG, "%s: negative M", fn);
    if (M > kMaxDim)
        return fail(MNB_ERR_SHAPE, "%s: M above 2^30", fn);
    if (M > 0 && N > 0 && (!X || !packed || !scales || !Y))
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL X, packed, scales or Y", fn);
    if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(Y, 16))
        return fail(MNB_ERR_ALIGN, "%s: X, packed and Y must be 16-byte aligned", fn);
    if (!aligned(scales, scale_t == MNB_F32 ? 4 : 2))
        return fail(MNB_ERR_ALIGN, "%s: scales misaligned", fn);
    return MNB_OK;
}

}  // namespace mnb

using namespace mnb;

extern "C" {

const char *mnb_last_error(void) { return g_msg; }

const char *mnb_version(void) { return "mnb 0.1 (sm_100a)"; }

int mnb_packed_sizes(int64_t N, int64_t K, int bs, mnb_dtype scale_t, int has_zp,
                     size_t *packed_bytes, size_t *scale_bytes, size_t *zp_bytes) {
    clear_error();
    int rc;
    if (!packed_bytes || !scale_bytes || !zp_bytes)
        return fail(MNB_ERR_INVALID_ARG, "mnb_packed_sizes: NULL output pointer");
    if ((rc = check_dtype("mnb_packed_sizes", "scale", scale_t)))
        return rc;
    if ((rc = check_weight_shape("mnb_packed_sizes", N, K, bs)))
        return rc;
    int64_t nb = K / bs;
    *packed_bytes = (size_t)(N * (K / 2));
    *scale_bytes = (size_t)(N * nb * (scale_t == MNB_F32 ? 4 : 2));
    *zp_bytes = has_zp ? (size_t)(N * ((nb + 1) / 2)) : 0;
    return MNB_OK;
}

int mnb_quantize_rtn(const float *W, int64_t N, int64_t K, int bs, int has_zp, uint8_t *packed,
                     void *scales, mnb_dtype scale_t, uint8_t *zp, void *stream) {
    clear_error();
    const char *fn = "mnb_quantize_rtn";
    int rc;
    if ((rc = check_dtype(fn, "scale", scale_t)) || (rc = check_weight_shape(fn, N, K, bs)))
        return rc;
    if (N == 0)
        return MNB_OK;
    if (!W || !packed || !scales || (has_zp && !zp))
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned(W, 16) || !aligned(packed, 16))
        return fail(MNB_ERR_ALIGN, "%s: W and packed must be 16-byte aligned", fn);
    if (!aligned(scales, scale_t == MNB_F32 ? 4 : 2))
        return fail(MNB_ERR_ALIGN, "%s: scales misaligned", fn);
    return launch_quantize_rtn(W, N, K, bs, has_zp ? 1 : 0, packed, scales, scale_t == MNB_F16,
                               has_zp ? zp : nullptr, (cudaStream_t)stream);
}

int mnb_dequantize(const uint8_t *packed, const void *scales, mnb_dtype scale_t, const uint8_t *zp,
                   int64_t N, int64_t K, int bs, void *W_out, mnb_dtype out_t, void *stream) {
    clear_error();
    const char *fn = "mnb_dequantize";
    int rc;
    if ((rc = check_dtype(fn, "scale", scale_t)) || (rc = check_dtype(fn, "output", out_t)) ||
        (rc = check_weight_shape(fn, N, K, bs)))
        return rc;
    if (N == 0)
        return MNB_OK;
    if (!packed || !scales || !W_out)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned(packed, 16) || !aligned(W_out, 16))
        return fail(MNB_ERR_ALIGN, "%s: packed and W_out must be 16-byte aligned", fn);
    if (!aligned(scales, scale_t == MNB_F32 ? 4 : 2))
        return fail(MNB_ERR_ALIGN, "%s: scales misaligned", fn);
    return launch_dequantize(packed, scales, scale_t == MNB_F16, zp, N, K, bs, W_out,
                             out_t == MNB_F16, (cudaStream_t)stream);
}

int mnb_gemv(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales,
             mnb_dtype scale_t, const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K,
             int bs, unsigned flags, void *stream) {
    clear_error();
    const char *fn = "mnb_gemv";
    int rc = check_matmul_args(fn, X, act_t, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (M > 32 || (M > 16 && act_t != MNB_F16))
        return fail(MNB_ERR_UNSUPPORTED, "%s: M=%lld above %d for %s activations (use mnb_gemm or mnb_matmul)", fn,
                    (long long)M, act_t == MNB_F16 ? 32 : 16, act_t == MNB_F16 ? "fp16" : "fp32");
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (M == 0 || N == 0)
        return MNB_OK;
    return launch_gemv(X, act_t == MNB_F16, packed, scales, scale_t == MNB_F16, zp, Y, (int)M,
                       (int)N, (int)K, bs, flags, (cudaStream_t)stream);
}

int mnb_gemv_swiglu(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                    const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, unsigned flags,
                    void *stream) {
    clear_error();
    const char *fn = "mnb_gemv_swiglu";
    int rc = check_matmul_args(fn, X, MNB_F16, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (M > 16)
        return fail(MNB_ERR_UNSUPPORTED, "%s: M=%lld > 16", fn, (long long)M);
    if (N % 16 != 0)
        return fail(MNB_ERR_SHAPE, "%s: N=%lld must be a multiple of 16 (8 gate + 8 up rows per group)", fn,
                    (long long)N);
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (M == 0 || N == 0)
        return MNB_OK;
    return launch_gemv_swiglu(X, packed, scales, scale_t == MNB_F16, zp, Y, (int)M, (int)N, (int)K, bs, flags,
                              (cudaStream_t)stream);
}

size_t mnb_gemv_argmax_workspace_bytes(int64_t M) {
    if (M < 1 || M > 16)
        return 0;
    return mnb::gemv_argmax_workspace_bytes((int)M);
}

int mnb_gemv_argmax(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                    const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, int32_t *ids,
                    float *max_out, void *workspace, size_t ws_bytes, unsigned flags, void *stream) {
    clear_error();
    const char *fn = "mnb_gemv_argmax";
    int rc = check_matmul_args(fn, X, MNB_F16, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (M < 1 || M > 16)
        return fail(MNB_ERR_UNSUPPORTED, "%s: M=%lld outside [1, 16]", fn, (long long)M);
    if (N < 1)
        return fail(MNB_ERR_SHAPE, "%s: N must be positive", fn);
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (!ids || !workspace)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL ids or workspace", fn);
    if (!aligned(ids, 4) || !aligned(max_out, 4) || !aligned(workspace, 16))
        return fail(MNB_ERR_ALIGN, "%s: ids / max_out need 4-byte, workspace 16-byte alignment", fn);
    const size_t need = mnb::gemv_argmax_workspace_bytes((int)M);
    if (ws_bytes < need)
        return fail(MNB_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, ws_bytes, need);
    return launch_gemv_argmax(X, packed, scales, scale_t == MNB_F16, zp, Y, (int)M, (int)N, (int)K, bs, ids,
                              max_out, workspace, flags, (cudaStream_t)stream);
}

int mnb_gemv_argmax_noalloc(const void *X, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
                            const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, int32_t *ids,
                            float *max_out, unsigned flags, void *stream) {
    clear_error();
    const char *fn = "mnb_gemv_argmax_noalloc";
    int rc = check_matmul_args(fn, X, MNB_F16, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (M < 1 || M > 16)
        return fail(MNB_ERR_UNSUPPORTED, "%s: M=%lld outside [1, 16]", fn, (long long)M);
    if (N < 1)
        return fail(MNB_ERR_SHAPE, "%s: N must be positive", fn);
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (!ids)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL ids", fn);
    if (!aligned(ids, 4) || !aligned(max_out, 4))
        return fail(MNB_ERR_ALIGN, "%s: ids and max_out need 4-byte alignment", fn);
    return launch_gemv_argmax_noalloc(X, packed, scales, scale_t == MNB_F16, zp, Y, (int)M, (int)N, (int)K, bs,
                                      ids, max_out, flags, (cudaStream_t)stream);
}

int mnb_gemm(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales,
             mnb_dtype scale_t, const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K,
             int bs, unsigned flags, void *stream) {
    clear_error();
    const char *fn = "mnb_gemm";
    int rc = check_matmul_args(fn, X, act_t, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (act_t != MNB_F16)
        return fail(MNB_ERR_UNSUPPORTED, "%s: the tensor-core path takes fp16 activations", fn);
    if (scale_t != MNB_F16)
        return fail(MNB_ERR_UNSUPPORTED, "%s: the tensor-core path takes fp16 scales (the q4f16 variant)", fn);
    if (N % 128 != 0 || K % 64 != 0)
        return fail(MNB_ERR_SHAPE, "%s: N=%lld must be a multiple of 128 and K=%lld of 64", fn,
                    (long long)N, (long long)K);
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (M == 0 || N == 0)
        return MNB_OK;
    return launch_gemm(X, packed, scales, scale_t == MNB_F16, zp, Y, (int)M, (int)N, (int)K, bs,
                       flags, (cudaStream_t)stream);
}

// Largest M the dispatcher serves with one decode GEMV launch before switching
// to the tensor-core GEMM (measured on the 1.7B decoder projections, per
// 196-projection pass: GEMV 1.84 / 2.16 / 2.53 ms against GEMM 2.51 / 2.51 /
// 2.51 ms at M = 17 / 24 / 28).
static const int64_t kGemvMaxM = 24;

int mnb_matmul(const void *X, mnb_dtype act_t, const uint8_t *packed, const void *scales, mnb_dtype scale_t,
               const uint8_t *zp, void *Y, int64_t M, int64_t N, int64_t K, int bs, unsigned flags, void *stream) {
    clear_error();
    const char *fn = "mnb_matmul";
    int rc = check_matmul_args(fn, X, act_t, packed, scales, scale_t, Y, M, N, K, bs);
    if (rc)
        return rc;
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    if (M == 0 || N == 0)
        return MNB_OK;
    const bool gemm_ok = act_t == MNB_F16 && scale_t == MNB_F16 && N % 128 == 0 && K % 64 == 0;
    if (gemm_ok && M > kGemvMaxM)
        return launch_gemm(X, packed, scales, scale_t == MNB_F16, zp, Y, (int)M, (int)N, (int)K, bs, flags,
                           (cudaStream_t)stream);
    // decode GEMV launches of up to 24 (fp16) or 16 (fp32) tokens; chunk
    // offsets are multiples of 8 rows, so every chunk keeps the 16-byte
    // alignment of X and Y
    const size_t elem = (act_t == MNB_F16) ? 2 : 4;
    const int64_t chunk = (act_t == MNB_F16) ? kGemvMaxM : 16;
    for (int64_t m0 = 0; m0 < M; m0 += chunk) {
        const int mc = (int)((M - m0 < chunk) ? (M - m0) : chunk);
        rc = launch_gemv(static_cast<const unsigned char *>(X) + (size_t)m0 * (size_t)K * elem, act_t == MNB_F16,
                         packed, scales, scale_t == MNB_F16, zp,
                         static_cast<unsigned char *>(Y) + (size_t)m0 * (size_t)N * elem, mc, (int)N, (int)K, bs,
                         flags, (cudaStream_t)stream);
        if (rc)
            return rc;
    }
    return MNB_OK;
}

int mnb_embed_gather(const int8_t *table, const float *row_scales, int64_t V, int64_t D,
                     const int32_t *ids, int64_t T, void *out, mnb_dtype out_t, int *status,
                     void *stream) {
    clear_error();
    const char *fn = "mnb_embed_gather";
    int rc;
    if ((rc = check_dtype(fn, "output", out_t)))
        return rc;
    if (V < 0 || D < 0 || T < 0)
        return fail(MNB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (D % 16 != 0 || D > kMaxDim || V > ((int64_t)1 << 31) - 1 || T > kMaxDim)
        return fail(MNB_ERR_SHAPE, "%s: D must be a multiple of 16; V < 2^31", fn);
    if (T == 0 || D == 0)
        return MNB_OK;
    if (!ids || !out || (V > 0 && (!table || !row_scales)))
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned(table, 16) || !aligned(out, 16) || !aligned(row_scales, 4) || !aligned(ids, 4) ||
        !aligned(status, 4))
        return fail(MNB_ERR_ALIGN, "%s: table and out must be 16-byte aligned", fn);
    return launch_embed_gather(table, row_scales, V, D, ids, T, out, out_t == MNB_F16, status,
                               (cudaStream_t)stream);
}

size_t mnb_gemv_chain_plan_bytes(int ntasks) { return gemv_chain_plan_bytes(ntasks); }

size_t mnb_gemv_chain_workspace_bytes(int ntasks) { return gemv_chain_workspace_bytes(ntasks); }

int mnb_gemv_chain_plan(const mnb_gemv_task *tasks, int ntasks, int64_t M, int bs, void *plan, size_t plan_bytes) {
    clear_error();
    static const char *fn = "mnb_gemv_chain_plan";
    if (!tasks || !plan)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL tasks or plan", fn);
    if (ntasks < 1 || ntasks > 65536)
        return fail(MNB_ERR_INVALID_ARG, "%s: ntasks=%d outside [1, 65536]", fn, ntasks);
    if (plan_bytes < gemv_chain_plan_bytes(ntasks))
        return fail(MNB_ERR_INVALID_ARG, "%s: plan buffer of %zu bytes, %zu needed", fn, plan_bytes,
                    gemv_chain_plan_bytes(ntasks));
    if (!aligned(plan, 64))
        return fail(MNB_ERR_ALIGN, "%s: plan buffer not 64-byte aligned", fn);
    if (bs != 32 && bs != 64)
        return fail(MNB_ERR_SHAPE, "%s: block size %d not in {32, 64}", fn, bs);
    if (M < 1)
        return fail(MNB_ERR_INVALID_ARG, "%s: M=%lld", fn, (long long)M);
    if (M > 8)
        return fail(MNB_ERR_UNSUPPORTED, "%s: M=%lld above 8", fn, (long long)M);
    return gemv_chain_plan(tasks, ntasks, (int)M, bs, plan, plan_bytes);
}

int mnb_gemv_chain(const void *plan, const void *plan_device, void *workspace, size_t ws_bytes, unsigned flags,
                   void *stream) {
    clear_error();
    static const char *fn = "mnb_gemv_chain";
    if (!plan || !plan_device || !workspace)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL plan, device plan or workspace", fn);
    if (!aligned(plan, 64) || !aligned(plan_device, 64) || !aligned(workspace, 4))
        return fail(MNB_ERR_ALIGN, "%s: plans must be 64-byte aligned, the workspace 4-byte aligned", fn);
    if (flags & ~(unsigned)MNB_FLAG_PDL)
        return fail(MNB_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, flags);
    return launch_gemv_chain(plan, plan_device, workspace, ws_bytes, flags, (cudaStream_t)stream);
}

static const int64_t kGptqMaxK = 8192;

int mnb_gptq_hessian(const void *X, mnb_dtype x_t, int64_t T, int64_t K, float *H, int accumulate, void *stream) {
    clear_error();
    const char *fn = "mnb_gptq_hessian";
    int rc;
    if ((rc = check_dtype(fn, "input", x_t)))
        return rc;
    if (T < 0 || K < 1 || K > kGptqMaxK)
        return fail(MNB_ERR_SHAPE, "%s: T=%lld, K=%lld (K must be in [1, %lld])", fn, (long long)T, (long long)K,
                    (long long)kGptqMaxK);
    if (T > kMaxDim)
        return fail(MNB_ERR_SHAPE, "%s: T above 2^30", fn);
    if (!H || (T > 0 && !X))
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL X or H", fn);
    if (!aligned(H, 4) || !aligned(X, x_t == MNB_F32 ? 4 : 2))
        return fail(MNB_ERR_ALIGN, "%s: X and H need their element alignment", fn);
    return launch_gptq_hessian(X, x_t == MNB_F16, T, K, H, accumulate ? 1 : 0, (cudaStream_t)stream);
}

size_t mnb_gptq_workspace_bytes(int64_t K) {
    if (K < 1 || K > kGptqMaxK)
        return 0;
    return gptq_workspace_bytes(K);
}

int mnb_gptq_prepare(const float *H, int64_t K, float percdamp, float *U, uint8_t *dead, void *workspace,
                     size_t ws_bytes, float *damp_used, void *stream) {
    clear_error();
    const char *fn = "mnb_gptq_prepare";
    if (K < 1 || K > kGptqMaxK)
        return fail(MNB_ERR_SHAPE, "%s: K=%lld outside [1, %lld]", fn, (long long)K, (long long)kGptqMaxK);
    if (!H || !U || !dead || !workspace)
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL H, U, dead or workspace", fn);
    if (!(percdamp >= 0.f) || !(percdamp <= 1.f))
        return fail(MNB_ERR_INVALID_ARG, "%s: percdamp %g outside [0, 1]", fn, (double)percdamp);
    if (!aligned(H, 4) || !aligned(U, 4) || !aligned(workspace, 16))
        return fail(MNB_ERR_ALIGN, "%s: H and U need 4-byte, the workspace 16-byte alignment", fn);
    if (ws_bytes < gptq_workspace_bytes(K))
        return fail(MNB_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, ws_bytes,
                    gptq_workspace_bytes(K));
    return launch_gptq_prepare(H, K, percdamp, U, dead, workspace, damp_used, (cudaStream_t)stream);
}

int mnb_gptq_quantize(const float *W, const float *U, const uint8_t *dead, int64_t N, int64_t K, int bs, int has_zp,
                      uint8_t *packed, void *scales, mnb_dtype scale_t, uint8_t *zp, void *stream) {
    clear_error();
    const char *fn = "mnb_gptq_quantize";
    int rc;
    if ((rc = check_dtype(fn, "scale", scale_t)) || (rc = check_weight_shape(fn, N, K, bs)))
        return rc;
    if (K > kGptqMaxK)
        return fail(MNB_ERR_SHAPE, "%s: K=%lld above %lld", fn, (long long)K, (long long)kGptqMaxK);
    if (N == 0)
        return MNB_OK;
    if (!W || !U || !packed || !scales || (has_zp && !zp))
        return fail(MNB_ERR_INVALID_ARG, "%s: NULL pointer", fn);
    if (!aligned(W, 4) || !aligned(U, 4) || !aligned(scales, scale_t == MNB_F32 ? 4 : 2))
        return fail(MNB_ERR_ALIGN, "%s: W, U and scales need their element alignment", fn);
    return launch_gptq_quantize(W, U, dead, N, K, bs, has_zp ? 1 : 0, packed, scales, scale_t == MNB_F16,
                                has_zp ? zp : nullptr, (cudaStream_t)stream);
}

int mnb_device_status(unsigned *status_out, int clear) {
    clear_error();
    if (!status_out)
        return fail(MNB_ERR_INVALID_ARG, "mnb_device_status: NULL output");
    *status_out = 0;
    const int rc = read_device_status(status_out, clear);
    if (rc)
        return rc;
    if (*status_out & 7u)   // bits 0-2: a bounded wait inside a kernel gave up
        return fail(MNB_ERR_TIMEOUT, "mnb_device_status: a device-side wait timed out (status 0x%x)", *status_out);
    return MNB_OK;
}

}  // extern "C"
