// internal.h -- launchers implemented in the kernel files, called by api.cu
// after the host-side argument checks.  Each returns an MNB_* status.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mnb.h"

namespace mnb {

int launch_quantize_rtn(const float *W, int64_t N, int64_t K, int bs, int has_zp, uint8_t *packed,
                        void *scales, int scale_f16, uint8_t *zp, cudaStream_t s);

int launch_dequantize(const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                      int64_t N, int64_t K, int bs, void *out, int out_f16, cudaStream_t s);

int launch_gemv(const void *X, int act_f16, const uint8_t *packed, const void *scales,
                int scale_f16, const uint8_t *zp, void *Y, int M, int N, int K, int bs,
                unsigned flags, cudaStream_t s);

int launch_gemv_tc(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                   void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s);

// One-token decode GEMV (fp16 activations and scales) whose CTAs hold their
// whole share of the weights in shared memory; returns 1 without launching
// anything for shapes it does not serve.  With ids != null it also does greedy
// decoding, with the workspace layout of mnb_gemv_argmax (256-byte counter
// header, then one (value, index) pair per CTA; at most two CTAs per SM); with
// swiglu != 0 the SwiGLU epilogue of mnb_gemv_swiglu.
int launch_gemv_resident(const void *X, const uint8_t *packed, const void *scales, const uint8_t *zp, void *Y, int N,
                         int K, int bs, unsigned flags, cudaStream_t s, int32_t *ids = nullptr,
                         float *max_out = nullptr, void *workspace = nullptr, int swiglu = 0);
// Whether one-token fp16 calls go to the resident kernel (tuning hook).
int gemv_resident_enabled();

// Decode GEMV with the SwiGLU epilogue over gate/up rows interleaved in 8-row groups.
int launch_gemv_swiglu(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                       void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s);

// Decode GEMV fused with greedy decoding (first maximum of each token's fp16 logits).
size_t gemv_argmax_workspace_bytes(int M);
int launch_gemv_argmax(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                       void *Y, int M, int N, int K, int bs, int32_t *ids, float *max_out, void *workspace,
                       unsigned flags, cudaStream_t s);

// The same with the scratch in a library-owned device array (no allocation).
size_t gemv_argmax_noalloc_capacity();
int launch_gemv_argmax_noalloc(const void *X, const uint8_t *packed, const void *scales, int scale_f16,
                               const uint8_t *zp, void *Y, int M, int N, int K, int bs, int32_t *ids,
                               float *max_out, unsigned flags, cudaStream_t s);

int launch_gemm(const void *X, const uint8_t *packed, const void *scales, int scale_f16,
                const uint8_t *zp, void *Y, int M, int N, int K, int bs, unsigned flags,
                cudaStream_t s);

int launch_embed_gather(const int8_t *table, const float *row_scales, int64_t V, int64_t D,
                        const int32_t *ids, int64_t T, void *out, int out_f16, int *status,
                        cudaStream_t s);

// A sequence of decode GEMVs as one persistent launch (plan on the host first).
size_t gemv_chain_plan_bytes(int ntasks);
size_t gemv_chain_workspace_bytes(int ntasks);
int gemv_chain_plan(const mnb_gemv_task *tasks, int ntasks, int M, int bs, void *plan, size_t plan_bytes);
int launch_gemv_chain(const void *plan, const void *plan_device, void *workspace, size_t ws_bytes, unsigned flags,
                      cudaStream_t s);

// GPTQ into the packed layout.
size_t gptq_workspace_bytes(int64_t K);
int launch_gptq_hessian(const void *X, int x_f16, int64_t T, int64_t K, float *H, int accumulate, cudaStream_t s);
int launch_gptq_prepare(const float *H, int64_t K, float percdamp, float *U, uint8_t *dead, void *workspace,
                        float *damp_used, cudaStream_t s);
int launch_gptq_quantize(const float *W, const float *U, const uint8_t *dead, int64_t N, int64_t K, int bs,
                         int has_zp, uint8_t *packed, void *scales, int scale_f16, uint8_t *zp, cudaStream_t s);

int read_device_status(unsigned *out, int clear);
int read_gemv_status(unsigned *out, int clear);     // ORs the decode kernel's word into *out
int read_res_status(unsigned *out, int clear);      // same for the one-token resident decode kernel
int read_chain_status(unsigned *out, int clear);    // the chain kernel's bits, shifted to bits 1-2

}  // namespace mnb
