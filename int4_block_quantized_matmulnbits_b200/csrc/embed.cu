// embed.cu -- int8 embedding-table lookup with one fp32 scale per row.
//
// "Qwen3-ASR-0.6B -- ONNX for the browser", "Pick a variant" ships the table as
// embed_tokens.int8.bin [151936, 1024] plus embed_scales.f32.bin [151936];
// "Building the prompt" step 4 forms each embedding as the int8 row times
// embed_scales[id], in fp32, or fp16 for the q4f16 graphs.  Here:
//   out[t][d] = round_out( fp32(table[id][d]) * row_scales[id] )
// with the product rounded to fp32 and, for fp16 output, rounded once more.
//
// HBM-bound gather: one warp per token, 16-byte loads of the int8 row and
// 16-byte stores of the output row.  Ids outside [0, V) give a zero row and an
// atomic OR of bit 0 into the optional status word; nothing traps.
#include "common.cuh"
#include "internal.h"

namespace mnb {

namespace {

template <bool OUT_F16>
__global__ void __launch_bounds__(256) embed_gather_kernel(const int8_t *__restrict__ table,
                                                           const float *__restrict__ row_scales,
                                                           int64_t V, int64_t D,
                                                           const int32_t *__restrict__ ids,
                                                           int64_t T, void *__restrict__ out,
                                                           int *__restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T)
        return;
    const int64_t id = ids[t];
    const bool ok = (id >= 0 && id < V);
    if (!ok && lane == 0 && status)
        atomicOr(status, 1);
    const float s = ok ? row_scales[id] : 0.f;
    const int8_t *row = table + (ok ? id : 0) * D;
    for (int64_t d = (int64_t)lane * 16; d < D; d += 32 * 16) {
        int8_t v[16];
        if (ok)
            *reinterpret_cast<uint4 *>(v) = ldg_v4(row + d);
        else
            *reinterpret_cast<uint4 *>(v) = make_uint4(0, 0, 0, 0);
        if (OUT_F16) {
            __half h[16];
#pragma unroll
            for (int i = 0; i < 16; i++)
                h[i] = __float2half_rn(__fmul_rn((float)v[i], s));
            uint4 *o = reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(out) + t * D + d);
            o[0] = reinterpret_cast<const uint4 *>(h)[0];
            o[1] = reinterpret_cast<const uint4 *>(h)[1];
        } else {
            float f[16];
#pragma unroll
            for (int i = 0; i < 16; i++)
                f[i] = __fmul_rn((float)v[i], s);
            float4 *o = reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + t * D + d);
#pragma unroll
            for (int i = 0; i < 4; i++)
                o[i] = reinterpret_cast<const float4 *>(f)[i];
        }
    }
}

}  // namespace

int launch_embed_gather(const int8_t *table, const float *row_scales, int64_t V, int64_t D,
                        const int32_t *ids, int64_t T, void *out, int out_f16, int *status,
                        cudaStream_t s) {
    const int64_t blocks = (T * 32 + 255) / 256;
    if (blocks > 0x7fffffff)
        return fail(MNB_ERR_SHAPE, "mnb_embed_gather: too many tokens");
    if (out_f16)
        embed_gather_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(table, row_scales, V, D, ids,
                                                                   T, out, status);
    else
        embed_gather_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(table, row_scales, V, D, ids,
                                                                    T, out, status);
    return check_launch("mnb_embed_gather");
}

}  // namespace mnb
