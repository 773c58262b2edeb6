// quantize.cu -- block-wise RTN quantization into the packed int4 layout, and
// the reverse dequantization.
//
// Quantization follows the recipe of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)",
// "Conversion details" (MatMulNBits, bits=4, block_size=32, is_symmetric=False)
// and the RTN variants of "Qwen3-ASR-0.6B -- ONNX for the browser" ("Pick a
// variant") and "qwen3-asr-0.6b-onnx-int4-merged" ("Provenance", block 64):
//   lo = min(0, min v), hi = max(0, max v), scale = (hi - lo) / 15,
//   zp = clamp(rint(-lo / scale), 0, 15), q = clamp(rint(v / scale + zp), 0, 15)
// with every operation an explicit IEEE round-to-nearest intrinsic, so the
// result is bit-identical to a scalar fp32 evaluation in the written order
// (divide, then add; rint rounds half to even).  Without zero points: scale =
// max|v| / 7, q = clamp(rint(v / scale) + 8, 0, 15).
//
// HBM-bound: reads 4 bytes per weight, writes ~0.58.  One unit of work is a PAIR
// of neighbouring blocks of one row (they share a zero-point byte); bs/4 lanes
// hold one block as float4s, so a warp's loads and stores are contiguous.
#include "common.cuh"
#include "internal.h"

namespace mnb {

namespace {

__device__ __forceinline__ int clamp15(int v) { return v < 0 ? 0 : (v > 15 ? 15 : v); }

template <int G>  // lanes per block: bs / 4
__global__ void __launch_bounds__(256) quantize_rtn_kernel(const float *__restrict__ W, int64_t N,
                                                           int64_t K, int has_zp,
                                                           uint8_t *__restrict__ packed,
                                                           void *__restrict__ scales, int scale_f16,
                                                           uint8_t *__restrict__ zp) {
    constexpr int BS = 4 * G;
    constexpr int UNITS_PER_WARP = 32 / (2 * G);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nb = K / BS;
    const int64_t zpb = (nb + 1) / 2;
    const int64_t units = N * zpb;

    const int64_t u = warp * UNITS_PER_WARP + lane / (2 * G);
    const int half = (lane / G) & 1;
    const int lg = lane % G;
    const int64_t n = u / zpb;
    const int64_t j = u - n * zpb;
    const int64_t b = 2 * j + half;
    const bool valid = (u < units) && (b < nb);

    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
        const float4 t = *reinterpret_cast<const float4 *>(W + n * K + b * BS + lg * 4);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }

    float s;
    int z;
    int q[4];
    if (has_zp) {
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            lo = fminf(lo, v[i]);
            hi = fmaxf(hi, v[i]);
        }
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
        z = 0;
        if (s != 0.f)
            z = clamp15(__float2int_rn(__fdiv_rn(-lo, s)));
#pragma unroll
        for (int i = 0; i < 4; i++) {
            q[i] = 0;
            if (s != 0.f)
                q[i] = clamp15(__float2int_rn(__fadd_rn(__fdiv_rn(v[i], s), (float)z)));
        }
    } else {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++)
            amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        s = __fdiv_rn(amax, 7.0f);
        z = 8;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            q[i] = 8;
            if (s != 0.f)
                q[i] = clamp15(__float2int_rn(__fdiv_rn(v[i], s)) + 8);
        }
    }

    // the odd block's zero point travels to the even block's first lane
    const int z_odd = __shfl_down_sync(0xffffffffu, z, G);
    if (!valid)
        return;
    const uint16_t two = (uint16_t)((q[0] | (q[1] << 4)) | ((q[2] | (q[3] << 4)) << 8));
    *reinterpret_cast<uint16_t *>(packed + n * (K / 2) + b * (BS / 2) + lg * 2) = two;
    if (lg == 0) {
        if (scale_f16)
            reinterpret_cast<__half *>(scales)[n * nb + b] = __float2half_rn(s);
        else
            reinterpret_cast<float *>(scales)[n * nb + b] = s;
        if (has_zp && half == 0) {
            const int hi_nib = (b + 1 < nb) ? z_odd : 0;
            zp[n * zpb + j] = (uint8_t)(z | (hi_nib << 4));
        }
    }
}

// One thread per 16 packed bytes (32 weights of one row).
template <bool OUT_F16>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t *__restrict__ packed,
                                                         const void *__restrict__ scales,
                                                         int scale_f16,
                                                         const uint8_t *__restrict__ zp, int64_t N,
                                                         int64_t K, int bs, void *__restrict__ out) {
    const int64_t chunks_per_row = K / 32;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= N * chunks_per_row)
        return;
    const int64_t n = idx / chunks_per_row;
    const int64_t k0 = (idx - n * chunks_per_row) * 32;
    const int64_t nb = K / bs;
    const int64_t b = k0 / bs;
    const uint4 p = *reinterpret_cast<const uint4 *>(packed + n * (K / 2) + k0 / 2);
    int z = 8;
    if (zp) {
        const uint8_t zb = zp[n * ((nb + 1) / 2) + b / 2];
        z = (b & 1) ? (zb >> 4) : (zb & 15);
    }
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    if (OUT_F16) {
        __half vals[32];
        if (scale_f16) {
            const float s = __half2float(reinterpret_cast<const __half *>(scales)[n * nb + b]);
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const int q = (words[i / 8] >> (4 * (i % 8))) & 15;
                vals[i] = __float2half_rn(__fmul_rn((float)(q - z), s));  // exact product
            }
        } else {
            const double s = (double)reinterpret_cast<const float *>(scales)[n * nb + b];
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const int q = (words[i / 8] >> (4 * (i % 8))) & 15;
                vals[i] = __double2half((double)(q - z) * s);  // exact product, one rounding
            }
        }
        uint4 *o = reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(out) + n * K + k0);
#pragma unroll
        for (int i = 0; i < 4; i++)
            o[i] = reinterpret_cast<const uint4 *>(vals)[i];
    } else {
        const float s = scale_f16 ? __half2float(reinterpret_cast<const __half *>(scales)[n * nb + b])
                                  : reinterpret_cast<const float *>(scales)[n * nb + b];
        float vals[32];
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const int q = (words[i / 8] >> (4 * (i % 8))) & 15;
            vals[i] = __fmul_rn((float)(q - z), s);
        }
        float4 *o = reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + n * K + k0);
#pragma unroll
        for (int i = 0; i < 8; i++)
            o[i] = reinterpret_cast<const float4 *>(vals)[i];
    }
}

}  // namespace

int launch_quantize_rtn(const float *W, int64_t N, int64_t K, int bs, int has_zp, uint8_t *packed,
                        void *scales, int scale_f16, uint8_t *zp, cudaStream_t s) {
    const int64_t nb = K / bs;
    const int64_t units = N * ((nb + 1) / 2);
    const int units_per_warp = (bs == 32) ? 2 : 1;
    const int64_t warps = (units + units_per_warp - 1) / units_per_warp;
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks > 0x7fffffff)
        return fail(MNB_ERR_SHAPE, "mnb_quantize_rtn: too many blocks");
    if (bs == 32)
        quantize_rtn_kernel<8><<<(unsigned)blocks, 256, 0, s>>>(W, N, K, has_zp, packed, scales,
                                                                scale_f16, zp);
    else
        quantize_rtn_kernel<16><<<(unsigned)blocks, 256, 0, s>>>(W, N, K, has_zp, packed, scales,
                                                                 scale_f16, zp);
    return check_launch("mnb_quantize_rtn");
}

int launch_dequantize(const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                      int64_t N, int64_t K, int bs, void *out, int out_f16, cudaStream_t s) {
    const int64_t threads = N * (K / 32);
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffff)
        return fail(MNB_ERR_SHAPE, "mnb_dequantize: too many blocks");
    if (out_f16)
        dequantize_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(packed, scales, scale_f16, zp, N,
                                                                 K, bs, out);
    else
        dequantize_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(packed, scales, scale_f16, zp,
                                                                  N, K, bs, out);
    return check_launch("mnb_dequantize");
}

}  // namespace mnb
