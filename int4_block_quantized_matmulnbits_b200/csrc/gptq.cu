// gptq.cu -- GPTQ quantization into the MatMulNBits layout ("Mega-ASR -- INT4
// ONNX (GPTQ-calibrated)", "Conversion details": algo=GPTQ, block_size=32,
// is_symmetric=False, bits=4; "GPTQ calibration": the Hessian accumulated from
// calibration activations, a Cholesky factorisation of its inverse, and the
// inner loop ported to the GPU in fp32, with a diagonal-jitter retry when the
// fp32 factorisation meets a barely-singular Hessian).
//
// The method is the published GPTQ (Frantar et al., 2022), column by column:
//   H = sum_t x_t x_t^T over calibration inputs; dead features (H_kk = 0) get
//   H_kk = 1 and zero weights; H += damp * mean(diag H) * I; U = the upper
//   Cholesky factor of H^-1 (H^-1 = U^T U).  Then for every weight row, for
//   i = 0 .. K-1: at a block's first column its scale and zero point come from
//   the row's current values of the block (the RTN rule of mnb_quantize_rtn);
//   q_i = RTN code of w_i; err = (w_i - (q_i - zp) s) / U_ii;
//   w_k -= err U_ik for k > i.
// Kernels:
//   gptq_hessian_kernel   64 x 64 tiles of H, fp32 accumulation over T.
//   gptq_damp_kernel      one CTA: dead features, the mean of the diagonal,
//                         the damped copy of H.
//   gptq_chol_step_kernel the factor H = R R^T with R UPPER triangular, one
//                         launch per column from the last to the first (the
//                         usual Cholesky with the index order reversed).  Then
//                         U = R^-1 is upper with U^T U = (R R^T)^-1 = H^-1: the
//                         factor GPTQ needs, without forming H^-1.
//   gptq_transpose_kernel R^T (stored by rows of the factor) -> R by rows.
//   gptq_trinv_kernel     U = R^-1, one warp per column, back substitution.
//   gptq_quantize_kernel  one warp per weight row: the row in shared memory,
//                         U's rows from L2, every update a separate fp32
//                         multiply and subtract in column order.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace mnb {

namespace {

// ---------------------------------------------------------------- H = X^T X

constexpr int kHT = 64;    // H tile
constexpr int kHS = 32;    // rows of X per stage

template <bool F16>
__global__ void __launch_bounds__(256) gptq_hessian_kernel(const void *X, int T, int K, float *H, int accumulate) {
    __shared__ float xi[kHS][kHT + 4];
    __shared__ float xj[kHS][kHT + 4];
    const int i0 = blockIdx.y * kHT, j0 = blockIdx.x * kHT;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < 4; b++) acc[a][b] = 0.f;
    for (int t0 = 0; t0 < T; t0 += kHS) {
        for (int e = threadIdx.x; e < kHS * kHT; e += 256) {
            const int r = e / kHT, col = e - r * kHT;
            const int t = t0 + r;
            float vi = 0.f, vj = 0.f;
            if (t < T) {
                if (F16) {
                    const __half *x = static_cast<const __half *>(X) + (int64_t)t * K;
                    if (i0 + col < K) vi = __half2float(x[i0 + col]);
                    if (j0 + col < K) vj = __half2float(x[j0 + col]);
                } else {
                    const float *x = static_cast<const float *>(X) + (int64_t)t * K;
                    if (i0 + col < K) vi = x[i0 + col];
                    if (j0 + col < K) vj = x[j0 + col];
                }
            }
            xi[r][col] = vi;
            xj[r][col] = vj;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < kHS; r++) {
            float a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                a[q] = xi[r][ty + 16 * q];
                b[q] = xj[r][tx + 16 * q];
            }
#pragma unroll
            for (int p = 0; p < 4; p++)
#pragma unroll
                for (int q = 0; q < 4; q++) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; p++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int i = i0 + ty + 16 * p, j = j0 + tx + 16 * q;
            if (i < K && j < K) {
                float *h = H + (int64_t)i * K + j;
                *h = accumulate ? *h + acc[p][q] : acc[p][q];
            }
        }
}

// ------------------------------------------------------- damping, dead columns

// One CTA of 1024 threads.  A = H with dead diagonal entries set to 1 and the
// diagonal raised by damp * mean(diag); dead[k] = (H_kk == 0).
__global__ void __launch_bounds__(1024) gptq_damp_kernel(const float *H, int K, float damp, float *A, uint8_t *dead,
                                                         int *info) {
    __shared__ float part[1024];
    float s = 0.f;
    for (int k = threadIdx.x; k < K; k += 1024) {
        const float d = H[(int64_t)k * K + k];
        s += (d == 0.f) ? 1.f : d;
    }
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w)
            part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    const float add = damp * (part[0] / (float)K);
    for (int k = threadIdx.x; k < K; k += 1024) {
        const float d = H[(int64_t)k * K + k];
        dead[k] = (d == 0.f) ? 1 : 0;
        A[(int64_t)k * K + k] = ((d == 0.f) ? 1.f : d) + add;
    }
    if (threadIdx.x == 0)
        *info = 0;
}

__global__ void gptq_copy_offdiag_kernel(const float *H, int K, float *A) {
    const int64_t n = (int64_t)K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
        if (e / K != e % K)
            A[e] = H[e];
}

// ------------------------------------------------ H = R R^T, R upper triangular

// Column j of R (rows i <= j), from the lower triangle of A (rows k, columns
// i <= k, updated in place): R_jj = sqrt(A_jj), R_ij = A_ji / R_jj, then
// A_ki -= R_ij R_kj for i <= k < j.  R^T is written by rows: Rt[j][i] = R_ij.
// Grid: 32 x 32 tiles (kb, ib) of the leading j x j block, ib <= kb.
__global__ void __launch_bounds__(256) gptq_chol_step_kernel(float *A, int K, int j, float *Rt, int *info) {
    const int ib = blockIdx.x, kb = blockIdx.y;
    if (ib > kb)
        return;
    const float d = A[(int64_t)j * K + j];
    if (!(d > 0.f) || !isfinite(d)) {   // not positive definite (in fp32)
        if (ib == 0 && kb == 0 && threadIdx.x == 0)
            atomicCAS(info, 0, j + 1);
        return;
    }
    const float r = sqrtf(d);
    __shared__ float ri[32], rk[32];
    const float *rowj = A + (int64_t)j * K;
    if (threadIdx.x < 32) {
        const int i = ib * 32 + threadIdx.x;
        ri[threadIdx.x] = (i < j) ? rowj[i] / r : 0.f;
    } else if (threadIdx.x < 64) {
        const int k = kb * 32 + threadIdx.x - 32;
        rk[threadIdx.x - 32] = (k < j) ? rowj[k] / r : 0.f;
    }
    __syncthreads();
    if (kb == ib) {   // the diagonal tiles also write R's column j, 32 rows each
        const int i = ib * 32 + (int)threadIdx.x;
        if (threadIdx.x < 32 && i < j)
            Rt[(int64_t)j * K + i] = ri[threadIdx.x];
        if (ib == 0 && threadIdx.x == 0)
            Rt[(int64_t)j * K + j] = r;
    }
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int i = ib * 32 + tx;
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const int kl = ty + 8 * q, k = kb * 32 + kl;
        if (k < j && i <= k) {
            float *a = A + (int64_t)k * K + i;
            *a = __fsub_rn(*a, __fmul_rn(ri[tx], rk[kl]));
        }
    }
}

// R (by rows) from Rt = R^T (by rows); zeros below the diagonal.
__global__ void gptq_transpose_kernel(const float *Rt, int K, float *R) {
    __shared__ float t[32][33];
    const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int q = ty; q < 32; q += 8) {
        const int y = y0 + q, x = x0 + tx;
        t[q][tx] = (y < K && x < K && x <= y) ? Rt[(int64_t)y * K + x] : 0.f;
    }
    __syncthreads();
    for (int q = ty; q < 32; q += 8) {
        const int y = x0 + q, x = y0 + tx;   // R[y][x] = Rt[x][y]
        if (y < K && x < K)
            R[(int64_t)y * K + x] = t[tx][q];
    }
}

// ------------------------------------------------------------- U = R^-1

// One warp per column j of U (upper): U_jj = 1 / R_jj, then for i = j-1 .. 0
// U_ij = -(sum_{m = i+1 .. j} R_im U_mj) / R_ii.  The column so far lives in
// the warp's shared memory; rows of R are read from L2.
__global__ void gptq_trinv_kernel(const float *R, int K, float *U) {
    extern __shared__ float col_smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int j = blockIdx.x * (blockDim.x >> 5) + wid;
    if (j >= K)
        return;
    float *col = col_smem + (size_t)wid * K;
    if (lane == 0)
        col[j] = 1.f / R[(int64_t)j * K + j];
    for (int i = j + 1 + lane; i < K; i += 32)
        U[(int64_t)i * K + j] = 0.f;
    __syncwarp();
    if (lane == 0)
        U[(int64_t)j * K + j] = col[j];
    for (int i = j - 1; i >= 0; i--) {
        const float *ri = R + (int64_t)i * K;
        float s = 0.f;
        for (int m = i + 1 + lane; m <= j; m += 32)
            s = fmaf(ri[m], col[m], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float v = -s / ri[i];
        if (lane == 0) {
            col[i] = v;
            U[(int64_t)i * K + j] = v;
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------- the column loop

__device__ __forceinline__ int clamp15(int v) { return v < 0 ? 0 : (v > 15 ? 15 : v); }

// One warp per row of W.  Every floating-point step is one IEEE operation in
// the order of the method's definition (no contraction into FMAs), so codes,
// scales and zero points do not depend on how the work is spread.
template <bool ZP>
__global__ void __launch_bounds__(256) gptq_quantize_kernel(const float *W, const float *U, const uint8_t *dead,
                                                            int N, int K, int bs, int warps, int scale_f16,
                                                            uint8_t *packed, void *scales, uint8_t *zp) {
    extern __shared__ float wsm[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int n = blockIdx.x * warps + wid;
    if (wid >= warps || n >= N)
        return;
    float *w = wsm + (size_t)wid * K;
    uint8_t *prow = reinterpret_cast<uint8_t *>(wsm + (size_t)warps * K) + (size_t)wid * (K / 2);
    const int nb = K / bs, zpb = (nb + 1) / 2;
    for (int k = lane; k < K; k += 32)
        w[k] = (dead && dead[k]) ? 0.f : W[(int64_t)n * K + k];
    __syncwarp();
    float s = 0.f;
    int z = ZP ? 0 : 8;
    uint32_t zbyte = 0;
    for (int i = 0; i < K; i++) {
        if (i % bs == 0) {
            // the block's scale and zero point from its current values
            const int b = i / bs;
            float lo = 0.f, hi = 0.f, amax = 0.f;
            for (int e = lane; e < bs; e += 32) {
                const float v = w[i + e];
                lo = fminf(lo, v);
                hi = fmaxf(hi, v);
                amax = fmaxf(amax, fabsf(v));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            }
            if (ZP) {
                s = __fdiv_rn(__fsub_rn(hi, lo), 15.f);
                z = (s != 0.f) ? clamp15((int)rintf(__fdiv_rn(-lo, s))) : 0;
                if (b & 1)
                    zbyte |= (uint32_t)z << 4;
                else
                    zbyte = (uint32_t)z;
                if (lane == 0 && ((b & 1) || b == nb - 1))
                    zp[(int64_t)n * zpb + b / 2] = (uint8_t)zbyte;
            } else {
                s = __fdiv_rn(amax, 7.f);
            }
            if (lane == 0) {
                if (scale_f16)
                    reinterpret_cast<__half *>(scales)[(int64_t)n * nb + b] = __float2half_rn(s);
                else
                    reinterpret_cast<float *>(scales)[(int64_t)n * nb + b] = s;
            }
        }
        const float wi = w[i];
        int q;
        if (ZP)
            q = (s != 0.f) ? clamp15((int)rintf(__fadd_rn(__fdiv_rn(wi, s), (float)z))) : 0;
        else
            q = (s != 0.f) ? clamp15((int)rintf(__fdiv_rn(wi, s)) + 8) : 8;
        if (lane == 0) {
            if (i & 1)
                prow[i >> 1] |= (uint8_t)(q << 4);
            else
                prow[i >> 1] = (uint8_t)q;
        }
        const float dq = __fmul_rn((float)(q - z), s);
        const float err = __fdiv_rn(__fsub_rn(wi, dq), U[(int64_t)i * K + i]);
        const float *ui = U + (int64_t)i * K;
        for (int k = i + 1 + lane; k < K; k += 32)
            w[k] = __fsub_rn(w[k], __fmul_rn(err, __ldg(ui + k)));
        __syncwarp();
    }
    for (int e = lane; e < K / 2; e += 32)
        packed[(int64_t)n * (K / 2) + e] = prow[e];
}

}  // namespace

size_t gptq_workspace_bytes(int64_t K) {
    return 2 * (size_t)K * (size_t)K * sizeof(float) + 256;
}

int launch_gptq_hessian(const void *X, int x_f16, int64_t T, int64_t K, float *H, int accumulate, cudaStream_t s) {
    const int tiles = (int)((K + kHT - 1) / kHT);
    dim3 grid((unsigned)tiles, (unsigned)tiles);
    if (x_f16)
        gptq_hessian_kernel<true><<<grid, 256, 0, s>>>(X, (int)T, (int)K, H, accumulate);
    else
        gptq_hessian_kernel<false><<<grid, 256, 0, s>>>(X, (int)T, (int)K, H, accumulate);
    return check_launch("mnb_gptq_hessian");
}

int launch_gptq_prepare(const float *H, int64_t K64, float percdamp, float *U, uint8_t *dead, void *workspace,
                        float *damp_used, cudaStream_t s) {
    const int K = (int)K64;
    float *A = static_cast<float *>(workspace);
    float *B = A + (size_t)K * K;                // R^T, then R
    int *info = reinterpret_cast<int *>(B + (size_t)K * K);
    const int tiles32 = (K + 31) / 32;
    // the pages' retry: a factorisation that meets a non-positive pivot in
    // fp32 starts again with ten times the damping (0.001 after none), up to
    // three times
    float damp = percdamp, tried = percdamp;
    for (int attempt = 0; attempt < 4; attempt++, tried = damp, damp = (damp > 0.f) ? damp * 10.f : 1e-3f) {
        gptq_copy_offdiag_kernel<<<296, 256, 0, s>>>(H, K, A);
        gptq_damp_kernel<<<1, 1024, 0, s>>>(H, K, damp, A, dead, info);
        for (int j = K - 1; j >= 0; j--) {
            const int t = (j + 31) / 32;   // tiles of the leading j x j block
            gptq_chol_step_kernel<<<dim3((unsigned)(t ? t : 1), (unsigned)(t ? t : 1)), 256, 0, s>>>(A, K, j, B,
                                                                                                   info);
        }
        int rc = check_launch("mnb_gptq_prepare");
        if (rc)
            return rc;
        int h_info = 0;
        cudaError_t e = cudaMemcpyAsync(&h_info, info, sizeof(int), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess)
            e = cudaStreamSynchronize(s);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gptq_prepare: %s", cudaGetErrorString(e));
        if (h_info != 0)
            continue;
        gptq_transpose_kernel<<<dim3((unsigned)tiles32, (unsigned)tiles32), 256, 0, s>>>(B, K, A);
        const int wpb = (K * 4 * 8 <= 96 * 1024) ? 8 : 4;   // warps per CTA: each holds a column of U
        const size_t smem = (size_t)wpb * K * sizeof(float);
        static int configured[kMaxDevices] = {};
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(gptq_trinv_kernel), (int)smem, configured);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gptq_prepare: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        gptq_trinv_kernel<<<(unsigned)((K + wpb - 1) / wpb), wpb * 32, smem, s>>>(A, K, U);
        if (damp_used)
            *damp_used = damp;
        return check_launch("mnb_gptq_prepare");
    }
    return fail(MNB_ERR_INVALID_ARG, "mnb_gptq_prepare: the Hessian is not positive definite in fp32 even with "
                                     "damping %g", (double)tried);
}

int launch_gptq_quantize(const float *W, const float *U, const uint8_t *dead, int64_t N, int64_t K, int bs,
                         int has_zp, uint8_t *packed, void *scales, int scale_f16, uint8_t *zp, cudaStream_t s) {
    // rows per CTA: each warp holds its row (K floats) and its packed bytes
    int warps = 8;
    while (warps > 1 && (size_t)warps * (K * 4 + K / 2) > 200 * 1024)
        warps >>= 1;
    const size_t smem = (size_t)warps * (K * 4 + K / 2);
    if (smem > 200 * 1024)
        return fail(MNB_ERR_SHAPE, "mnb_gptq_quantize: K=%lld too large", (long long)K);
    const unsigned grid = (unsigned)((N + warps - 1) / warps);
    static int configured[2][kMaxDevices] = {};
    auto fn = has_zp ? gptq_quantize_kernel<true> : gptq_quantize_kernel<false>;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(fn), (int)smem, configured[has_zp ? 1 : 0]);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gptq_quantize: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    fn<<<grid, 256, smem, s>>>(W, U, dead, (int)N, (int)K, bs, warps, scale_f16, packed, scales, zp);
    return check_launch("mnb_gptq_quantize");
}

}  // namespace mnb
