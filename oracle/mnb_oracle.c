/*
 * mnb_oracle.c -- plain, slow, obviously correct CPU oracle for the MatMulNBits
 * operator (weight-only 4-bit block quantization).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * Compiled with -O2 -ffp-contract=off (no FMA contraction, no fast-math), so
 * every float expression below is evaluated as written, one IEEE operation at a
 * time, in the precision written.
 *
 * What the operator is (sources, by page title and section):
 *   - "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", intro and "Conversion details":
 *     MatMulNBits, 4 bits, block_size=32, is_symmetric=False (asymmetric, one
 *     zero point per block), weight-only.
 *   - "int4 STT weights for sherpa-onnx", "Why int4 rather than the usual
 *     int8": weight-only, in blocks, activations untouched.
 *   - "Qwen3-ASR-0.6B -- ONNX for the browser", "Pick a variant": RTN, block 32;
 *     q4 keeps float tensors fp32, q4f16 keeps them fp16.
 *   - "qwen3-asr-0.6b-onnx-int4-merged", "Provenance": RTN, block_size=64.
 *   - "Qwen3-ASR-0.6B -- ONNX for the browser", "Building the prompt" step 4:
 *     embedding = row of the int8 table times embed_scales[id] -> fp32/fp16.
 *
 * The pages never write the arithmetic down.  The definitions used here are the
 * standard asymmetric int4 ones:
 *     w = (q - zp) * scale,   zp = 8 when no zero-point tensor is given,
 *     Y[m, n] = sum_k X[m, k] * w[n, k]           (Y = X . dequant(W)^T)
 *     RTN:  scale = (max - min) / 15,  zp = clamp(round(-min / scale), 0, 15),
 *           q = clamp(round(v / scale + zp), 0, 15).
 * Readings of points the pages leave open (each also listed in the design notes):
 *   R1 nibble order: element 2j of a row sits in the LOW nibble of byte j,
 *      element 2j+1 in the high nibble; the zero point of block b sits in byte
 *      b/2 of its row, low nibble when b is even.
 *   R2 layout: packed [N][K/2] bytes (= [N][K/bs][bs/2]), scales [N][K/bs],
 *      zero points [N][ceil((K/bs)/2)] bytes, all row-major, odd tail nibble 0.
 *   R3 the RTN range includes zero: lo = min(0, min v), hi = max(0, max v).
 *   R4 round() is round-half-to-even (rintf in the default rounding mode).
 *   R5 q = rint( fl( fl(v / scale) + zp ) ): an IEEE division, then an add.
 *   R6 scale == 0 (an all-zero block): zp = 0, q = 0.
 *   R7 fp16 scales: quantize with the fp32 scale, then store fp16_rn(scale).
 *   R8 no-zero-point (symmetric) variant: zp = 8, scale = absmax / 7,
 *      q = clamp(rint(v / scale) + 8, 0, 15); scale == 0 -> q = 8.
 *      PARITY UNPINNED by the pages (they only show is_symmetric=False).
 *   R9 embedding value = fp16_rn( fp32( fp32(int8) * fp32(row_scale) ) ).
 *
 * GPTQ ("Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", "Conversion details":
 * algo=GPTQ, block_size=32, is_symmetric=False; "GPTQ calibration": Hessian
 * accumulated from calibration activations, Cholesky factorisation of its
 * inverse, the inner loop run in fp32 on the GPU).  The pages name the method
 * and do not print it; this is the published algorithm (Frantar et al.,
 * "GPTQ: Accurate Post-Training Quantization for Generative Pre-trained
 * Transformers", 2022), column by column without its lazy batching:
 *     for each row, for i = 0 .. K-1:
 *         at the first column of a block, the block's scale and zero point
 *             from the row's CURRENT values of that block (RTN rule above);
 *         q_i = the RTN code of w_i;  err = (w_i - (q_i - zp) * scale) / U[i][i];
 *         w_k -= err * U[i][k]  for every k > i,
 *     with U the upper Cholesky factor of H^-1 (H^-1 = U^T U).
 *   R10 the block parameters use the weights as updated by every earlier column
 *       (the lazy-batch implementations read them as of their last batch
 *       boundary, a scheduling artefact not adopted here).
 *   R11 codes, scales and zero points follow R1-R8 exactly (the same quantizer
 *       as RTN), computed from the fp32 scale; fp16 scales are stored rounded
 *       after the loop (R7).  The loop runs in fp32, the precision of the pages'
 *       GPU port, one IEEE operation at a time in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_BAD (-1)

/* ---- nibble access (reading R1) ------------------------------------------ */

static int nibble_get(const uint8_t *row, int64_t i)
{
    uint8_t byte = row[i / 2];
    if (i % 2 == 0)
        return byte & 0x0F;
    return (byte >> 4) & 0x0F;
}

static void nibble_set(uint8_t *row, int64_t i, int v)
{
    uint8_t byte = row[i / 2];
    if (i % 2 == 0)
        byte = (uint8_t)((byte & 0xF0) | (v & 0x0F));
    else
        byte = (uint8_t)((byte & 0x0F) | ((v & 0x0F) << 4));
    row[i / 2] = byte;
}

static int clamp_0_15(int v)
{
    if (v < 0)
        return 0;
    if (v > 15)
        return 15;
    return v;
}

/* ---- sizes of the packed layout (reading R2) ------------------------------ */

/* Bytes of the three tensors for one [N, K] weight.  scale_bytes is 4 (fp32)
 * or 2 (fp16); has_zp = 0 means no zero-point tensor. */
int orc_packed_sizes(int64_t N, int64_t K, int64_t bs, int64_t scale_bytes, int has_zp,
                     int64_t *packed_bytes, int64_t *scale_bytes_out, int64_t *zp_bytes)
{
    if (N < 0 || K <= 0 || bs <= 0 || K % bs != 0 || bs % 2 != 0)
        return ORC_BAD;
    int64_t nb = K / bs;
    *packed_bytes = N * (K / 2);
    *scale_bytes_out = N * nb * scale_bytes;
    *zp_bytes = has_zp ? N * ((nb + 1) / 2) : 0;
    return ORC_OK;
}

/* ---- RTN quantization ------------------------------------------------------ */

/* W: fp32 [N][K].  Writes packed [N][K/2], scales [N][nb] (fp32, or fp16 when
 * scale_f16), and zp [N][ceil(nb/2)] when has_zp (else zp may be NULL). */
int orc_quantize_rtn(const float *W, int64_t N, int64_t K, int64_t bs, int has_zp,
                     int scale_f16, uint8_t *packed, void *scales, uint8_t *zp)
{
    if (N < 0 || K <= 0 || bs <= 0 || K % bs != 0 || bs % 2 != 0)
        return ORC_BAD;
    int64_t nb = K / bs;
    int64_t zp_row = (nb + 1) / 2;
    memset(packed, 0, (size_t)(N * (K / 2)));
    if (has_zp)
        memset(zp, 0, (size_t)(N * zp_row));

    for (int64_t n = 0; n < N; n++) {
        uint8_t *prow = packed + n * (K / 2);
        for (int64_t b = 0; b < nb; b++) {
            const float *v = W + n * K + b * bs;
            float s;
            int z;
            if (has_zp) {
                /* reading R3: the range [lo, hi] always contains zero */
                float lo = 0.0f, hi = 0.0f;
                for (int64_t i = 0; i < bs; i++) {
                    if (v[i] < lo)
                        lo = v[i];
                    if (v[i] > hi)
                        hi = v[i];
                }
                s = (hi - lo) / 15.0f;
                z = 0;
                if (s != 0.0f)
                    z = clamp_0_15((int)rintf(-lo / s));
                for (int64_t i = 0; i < bs; i++) {
                    int q = 0;
                    if (s != 0.0f) {
                        float t = v[i] / s;       /* reading R5: divide ... */
                        t = t + (float)z;         /* ... then add zp        */
                        q = clamp_0_15((int)rintf(t));
                    }
                    nibble_set(prow, b * bs + i, q);
                }
                nibble_set(zp + n * zp_row, b, z);
            } else {
                /* reading R8 (symmetric, implicit zp = 8) */
                float amax = 0.0f;
                for (int64_t i = 0; i < bs; i++) {
                    float a = fabsf(v[i]);
                    if (a > amax)
                        amax = a;
                }
                s = amax / 7.0f;
                for (int64_t i = 0; i < bs; i++) {
                    int q = 8;
                    if (s != 0.0f)
                        q = clamp_0_15((int)rintf(v[i] / s) + 8);
                    nibble_set(prow, b * bs + i, q);
                }
            }
            if (scale_f16)
                ((_Float16 *)scales)[n * nb + b] = (_Float16)s;   /* reading R7 */
            else
                ((float *)scales)[n * nb + b] = s;
        }
    }
    return ORC_OK;
}

/* ---- GPTQ quantization (readings R10, R11) -------------------------------- */

/* W: fp32 [N][K] (read only).  U: fp32 [K][K], row-major upper Cholesky factor
 * of the (damped) inverse Hessian; only U[i][k] with k >= i is read.  dead:
 * K flags or NULL; a dead input feature's weights are zeroed before the loop.
 * Outputs as orc_quantize_rtn. */
int orc_gptq_quantize(const float *W, const float *U, const uint8_t *dead, int64_t N, int64_t K, int64_t bs,
                      int has_zp, int scale_f16, uint8_t *packed, void *scales, uint8_t *zp)
{
    if (N < 0 || K <= 0 || bs <= 0 || K % bs != 0 || bs % 2 != 0)
        return ORC_BAD;
    int64_t nb = K / bs;
    int64_t zp_row = (nb + 1) / 2;
    memset(packed, 0, (size_t)(N * (K / 2)));
    if (has_zp)
        memset(zp, 0, (size_t)(N * zp_row));
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t n = 0; n < N; n++) {
        float *w = (float *)malloc((size_t)K * sizeof(float));
        if (!w) {
            bad = 1;
            continue;
        }
        for (int64_t k = 0; k < K; k++)
            w[k] = (dead && dead[k]) ? 0.0f : W[n * K + k];
        uint8_t *prow = packed + n * (K / 2);
        float s = 0.0f;
        int z = 0;
        for (int64_t i = 0; i < K; i++) {
            if (i % bs == 0) {
                /* the block's parameters from its current values */
                int64_t b = i / bs;
                const float *v = w + i;
                if (has_zp) {
                    float lo = 0.0f, hi = 0.0f;   /* R3 */
                    for (int64_t j = 0; j < bs; j++) {
                        if (v[j] < lo)
                            lo = v[j];
                        if (v[j] > hi)
                            hi = v[j];
                    }
                    s = (hi - lo) / 15.0f;
                    z = 0;
                    if (s != 0.0f)
                        z = clamp_0_15((int)rintf(-lo / s));
                    nibble_set(zp + n * zp_row, b, z);
                } else {
                    float amax = 0.0f;   /* R8 */
                    for (int64_t j = 0; j < bs; j++) {
                        float a = fabsf(v[j]);
                        if (a > amax)
                            amax = a;
                    }
                    s = amax / 7.0f;
                    z = 8;
                }
                if (scale_f16)
                    ((_Float16 *)scales)[n * nb + b] = (_Float16)s;
                else
                    ((float *)scales)[n * nb + b] = s;
            }
            int q;
            if (has_zp) {
                q = 0;
                if (s != 0.0f) {
                    float t = w[i] / s;   /* R5 */
                    t = t + (float)z;
                    q = clamp_0_15((int)rintf(t));
                }
            } else {
                q = 8;
                if (s != 0.0f)
                    q = clamp_0_15((int)rintf(w[i] / s) + 8);
            }
            nibble_set(prow, i, q);
            /* error feedback through row i of U */
            float dq = (float)(q - z) * s;
            float err = (w[i] - dq) / U[i * K + i];
            for (int64_t k = i + 1; k < K; k++)
                w[k] = w[k] - err * U[i * K + k];
        }
        free(w);
    }
    return bad ? ORC_BAD : ORC_OK;
}

/* ---- dequantization --------------------------------------------------------- */

static double scale_at(const void *scales, int scale_f16, int64_t idx)
{
    if (scale_f16)
        return (double)((const _Float16 *)scales)[idx];
    return (double)((const float *)scales)[idx];
}

static int zp_at(const uint8_t *zp, int64_t zp_row, int64_t n, int64_t b)
{
    if (zp == NULL)
        return 8;                 /* no zero-point tensor: zp = 8 */
    return nibble_get(zp + n * zp_row, b);
}

/* w[n][k] = (q - zp) * scale, exact in double (a 5-bit integer times a 24-bit
 * significand).  out_kind: 0 = double, 1 = fp32 (one rounding), 2 = fp16 (one
 * rounding). */
int orc_dequantize(const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                   int64_t N, int64_t K, int64_t bs, int out_kind, void *out)
{
    if (N < 0 || K <= 0 || bs <= 0 || K % bs != 0 || bs % 2 != 0)
        return ORC_BAD;
    int64_t nb = K / bs;
    int64_t zp_row = (nb + 1) / 2;
    for (int64_t n = 0; n < N; n++) {
        const uint8_t *prow = packed + n * (K / 2);
        for (int64_t k = 0; k < K; k++) {
            int64_t b = k / bs;
            int q = nibble_get(prow, k);
            int z = zp_at(zp, zp_row, n, b);
            double w = (double)(q - z) * scale_at(scales, scale_f16, n * nb + b);
            if (out_kind == 0)
                ((double *)out)[n * K + k] = w;
            else if (out_kind == 1)
                ((float *)out)[n * K + k] = (float)w;
            else
                ((_Float16 *)out)[n * K + k] = (_Float16)w;
        }
    }
    return ORC_OK;
}

/* ---- the matmul: Y = X . dequant(W)^T ------------------------------------- */

/* X: double [M][K] (the activations, converted exactly from fp32 or fp16).
 * cols: the output columns n to compute (NULL = all N, in order); Y: double
 * [M][ncols].  Triple loop, double accumulation in k order. */
int orc_matmul(const double *X, int64_t M, int64_t K, const uint8_t *packed, const void *scales,
               int scale_f16, const uint8_t *zp, int64_t N, int64_t bs, const int64_t *cols,
               int64_t ncols, double *Y)
{
    if (M < 0 || N < 0 || K <= 0 || bs <= 0 || K % bs != 0 || bs % 2 != 0)
        return ORC_BAD;
    int64_t nb = K / bs;
    int64_t zp_row = (nb + 1) / 2;
    if (cols == NULL)
        ncols = N;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
    for (int64_t j = 0; j < ncols; j++) {
        int64_t n = cols ? cols[j] : j;
        if (n < 0 || n >= N) {
            bad = 1;
            continue;
        }
        const uint8_t *prow = packed + n * (K / 2);
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                int64_t b = k / bs;
                int q = nibble_get(prow, k);
                int z = zp_at(zp, zp_row, n, b);
                double w = (double)(q - z) * scale_at(scales, scale_f16, n * nb + b);
                acc += X[m * K + k] * w;
            }
            Y[m * ncols + j] = acc;
        }
    }
    return bad ? ORC_BAD : ORC_OK;
}

/* ---- int8 embedding gather (reading R9) ------------------------------------ */

/* out[t][d] = row_scales[id] * table[id][d] (fp32 product, then fp16 when
 * out_f16).  An id outside [0, V) gives a zero row and sets bit 0 of the
 * returned status. */
int orc_embed_gather(const int8_t *table, const float *row_scales, int64_t V, int64_t D,
                     const int32_t *ids, int64_t T, int out_f16, void *out)
{
    int status = 0;
    for (int64_t t = 0; t < T; t++) {
        int64_t id = ids[t];
        int ok = (id >= 0 && id < V);
        if (!ok)
            status |= 1;
        for (int64_t d = 0; d < D; d++) {
            float v = 0.0f;
            if (ok)
                v = (float)table[id * D + d] * row_scales[id];
            if (out_f16)
                ((_Float16 *)out)[t * D + d] = (_Float16)v;
            else
                ((float *)out)[t * D + d] = v;
        }
    }
    return status;
}

/* Number of threads the parallel loop above uses. */
int orc_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
