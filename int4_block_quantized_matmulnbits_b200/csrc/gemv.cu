// gemv.cu -- decode-shaped MatMulNBits, Y[M][N] = X[M][K] . dequant(W)^T with
// 1 <= M <= 16 (the per-token decoder_step of "Qwen3-ASR-0.6B -- ONNX for the
// browser", "Graph contracts", and of "Mega-ASR -- INT4 ONNX", "What's in this
// repo": decoder_step_int4).
//
// This is HBM-bound: every packed byte is read exactly once, so the kernel is
// built around moving weight bytes.
//   * CTA = 4 warps over a tile of 16 weight rows.  Thread (g = lane/4, c =
//     lane%4) owns rows g and g+8; a warp walks "super-chunks" of 128 k, in
//     which thread c loads the 16-byte chunk c (32 nibbles, one block of 32 or
//     half a block of 64) of both rows with 128-bit streaming loads.  The warp's
//     four loads of a row are one contiguous 64-byte segment.
//   * Weights are prefetched into a register ring several super-chunks deep,
//     and the first loads are issued BEFORE griddepcontrol.wait, so under
//     programmatic dependent launch the weight stream of this kernel overlaps
//     the tail of the previous one; X is read only after the wait.
//   * When the row tiles alone cannot fill the 148 SMs, K is split over a
//     thread-block cluster of S CTAs; the partial sums meet in distributed
//     shared memory (no global scratch, no second kernel, no atomics).
//   * X for the CTA's K range is staged once in shared memory, permuted so one
//     16-byte load yields the activation pairs that match the dequantized
//     weight pairs.
// Unpack + dequant happen in registers: (mask | 0x6400) turns a nibble q into
// the fp16 1024+q exactly, and one half2 subtract (or fma for the high nibble,
// 1024+16q) leaves the exact q - zp.  Two inner products:
//   MMA (fp16 activations): the weight half2s are scaled to
//     fp16_rn((q - zp) * scale) and fed to mma.sync m16n8k16 with fp32
//     accumulation; the 16 rows are the MMA's M, the tokens its N (8 or 16).
//     This keeps the multiply-adds off the CUDA cores, whose issue slots the
//     unpack already fills.
//   CC (fp32 activations, and an fp16 variant): CUDA-core FMAs, fp32 partial
//     per chunk, times the scale, summed in fp32, reduced across the 4 lanes of
//     a row with warp shuffles.
#include "common.cuh"
#include "internal.h"

namespace mnb {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;
constexpr int kPF = 4;            // super-chunks in flight per warp
constexpr int kSuper = 128;       // k per super-chunk
constexpr int kMaxCluster = 8;

enum { MODE_MMA = 0, MODE_CC = 1 };

struct Params {
    const void *X;
    const uint8_t *packed;
    const void *scales;
    const uint8_t *zp;
    void *Y;
    int M, N, K;
    int bs_shift;   // log2(bs) - 5
    int nb, zpb;
    int scale_f16;
    int S;          // CTAs per cluster (K splits)
    int ks;         // k per split, multiple of kSuper
    int nsc;        // super-chunks per split
    int xs_stride;  // bytes per token row of the staged X
};

struct Slot {
    uint4 p0, p1;      // 32 nibbles of row g and of row g+8
    uint32_t s0, s1;   // raw scale bits (fp16 in the low half, or fp32)
    uint32_t z0, z1;   // zero point nibble (8 when absent)
};

__device__ __forceinline__ Slot load_slot(const Params &p, int row0, int kbeg, int sc, int c) {
    Slot s;
    s.p0 = s.p1 = make_uint4(0, 0, 0, 0);
    s.s0 = s.s1 = 0;
    s.z0 = s.z1 = 8;
    const int k0 = kbeg + sc * kSuper + c * 32;
    if (sc >= p.nsc || k0 >= p.K)
        return s;
    const int blk = k0 >> (5 + p.bs_shift);
    const int rows[2] = {row0, row0 + 8};
#pragma unroll
    for (int r = 0; r < 2; r++) {
        const int n = rows[r];
        if (n >= p.N)
            continue;
        const uint4 v = ldg_stream_v4(p.packed + (int64_t)n * (p.K / 2) + k0 / 2);
        uint32_t sb;
        if (p.scale_f16)
            sb = __ldg(reinterpret_cast<const unsigned short *>(p.scales) + (int64_t)n * p.nb + blk);
        else
            sb = __float_as_uint(__ldg(reinterpret_cast<const float *>(p.scales) + (int64_t)n * p.nb + blk));
        uint32_t z = 8;
        if (p.zp) {
            const uint32_t zb = __ldg(p.zp + (int64_t)n * p.zpb + (blk >> 1));
            z = (blk & 1) ? (zb >> 4) : (zb & 15);
        }
        if (r == 0) { s.p0 = v; s.s0 = sb; s.z0 = z; }
        else        { s.p1 = v; s.s1 = sb; s.z1 = z; }
    }
    return s;
}

// 8 nibbles -> 4 half2 of exact (q - zp): (e0,e4), (e1,e5), (e2,e6), (e3,e7).
__device__ __forceinline__ void dq_word(uint32_t w, uint32_t Z, uint32_t Zhi, uint32_t out[4]) {
    const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    const uint32_t lo0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
    const uint32_t hi0 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
    const uint32_t w8 = w >> 8;
    const uint32_t lo1 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
    const uint32_t hi1 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
    out[0] = h2_as_u32(__hsub2(u32_as_h2(lo0), u32_as_h2(Z)));
    out[1] = h2_as_u32(__hfma2(u32_as_h2(hi0), sixteenth, u32_as_h2(Zhi)));
    out[2] = h2_as_u32(__hsub2(u32_as_h2(lo1), u32_as_h2(Z)));
    out[3] = h2_as_u32(__hfma2(u32_as_h2(hi1), sixteenth, u32_as_h2(Zhi)));
}

// 16 half2 of exact (q - zp) for one 16-byte chunk; element order per word as dq_word.
__device__ __forceinline__ void dq_chunk(const uint4 &p, uint32_t z, uint32_t out[16]) {
    const uint32_t Z = 0x64006400u | (z * 0x00010001u);          // 1024 + zp
    const uint32_t Zhi = 0xD400D400u + (z * 0x00100010u);        // -(64 + zp)
    dq_word(p.x, Z, Zhi, out + 0);
    dq_word(p.y, Z, Zhi, out + 4);
    dq_word(p.z, Z, Zhi, out + 8);
    dq_word(p.w, Z, Zhi, out + 12);
}

__device__ __forceinline__ float scale_f32(uint32_t raw, int f16) {
    return f16 ? __half2float(__ushort_as_half((unsigned short)raw)) : __uint_as_float(raw);
}

__device__ __forceinline__ half2 scale_h2(uint32_t raw, int f16) {
    const __half h = f16 ? __ushort_as_half((unsigned short)raw) : __float2half_rn(__uint_as_float(raw));
    return __halves2half2(h, h);
}

__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// MP: tokens held per thread (MMA: 8 or 16, CC: 1, 2, 4, 8 or 16).
template <int MODE, bool ACT_F16, int MP>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int rank = (p.S > 1) ? (int)cluster_ctarank() : 0;
    const int tile = blockIdx.x / p.S;
    const int row0 = tile * kRows + g;
    const int kbeg = rank * p.ks;

    unsigned char *xs = smem;                                                   // [MP][xs_stride]
    float *red = reinterpret_cast<float *>(smem + MP * p.xs_stride);            // [kWarps][16][MP]
    float *part = red + kWarps * kRows * MP;                                    // [16][MP]

    // ---- weights first: they do not depend on the previous kernel
    Slot ring[kPF];
#pragma unroll
    for (int i = 0; i < kPF; i++)
        ring[i] = load_slot(p, row0, kbeg, warp + i * kWarps, c);
    pdl_launch_dependents();
    pdl_wait();

    // ---- stage X[:, kbeg : kbeg + ks) (zero-padded to MP tokens and the split)
    if (ACT_F16) {
        const __half *X = reinterpret_cast<const __half *>(p.X);
        const int units = MP * p.nsc * 16;                      // 16-byte units of 8 halves
        for (int u = tid; u < units; u += kThreads) {
            const int m = u / (p.nsc * 16);
            const int r = u - m * p.nsc * 16;
            const int sc = r >> 4, cc = (r >> 2) & 3, w = r & 3;
            const int k = kbeg + sc * kSuper + cc * 32 + w * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < p.M && k < p.K)
                v = ldg_v4(X + (int64_t)m * p.K + k);
            uint4 o;   // (x0,x4) (x1,x5) (x2,x6) (x3,x7)
            o.x = __byte_perm(v.x, v.z, 0x5410);
            o.y = __byte_perm(v.x, v.z, 0x7632);
            o.z = __byte_perm(v.y, v.w, 0x5410);
            o.w = __byte_perm(v.y, v.w, 0x7632);
            *reinterpret_cast<uint4 *>(xs + m * p.xs_stride + sc * 256 + w * 64 + cc * 16) = o;
        }
    } else {
        const float *X = reinterpret_cast<const float *>(p.X);
        const int units = MP * p.nsc * 32;                      // 16-byte units of 4 floats
        for (int u = tid; u < units; u += kThreads) {
            const int m = u / (p.nsc * 32);
            const int r = u - m * p.nsc * 32;
            const int sc = r >> 5, cc = (r >> 3) & 3, j = r & 7;
            const int k = kbeg + sc * kSuper + cc * 32 + j * 4;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < p.M && k < p.K)
                v = ldg_v4(X + (int64_t)m * p.K + k);
            *reinterpret_cast<uint4 *>(xs + m * p.xs_stride + sc * 512 + j * 64 + cc * 16) = v;
        }
    }
    __syncthreads();

    // ---- main loop over this warp's super-chunks
    constexpr int NT = (MODE == MODE_MMA) ? MP / 8 : 1;
    float accm[NT][4];                        // MMA accumulators
    float accc[2][MP];                        // CC accumulators: rows g, g+8 x tokens
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int i = 0; i < 4; i++) accm[t][i] = 0.f;
#pragma unroll
    for (int r = 0; r < 2; r++)
#pragma unroll
        for (int m = 0; m < MP; m++) accc[r][m] = 0.f;

    const uint32_t xs_base = smem_u32(xs);
    const int nmine = (p.nsc > warp) ? (p.nsc - warp + kWarps - 1) / kWarps : 0;
    for (int base = 0; base < nmine; base += kPF) {
#pragma unroll
        for (int i = 0; i < kPF; i++) {
            const int it = base + i;
            if (it < nmine) {
                const Slot cur = ring[i];
                const int sc = warp + it * kWarps;
                ring[i] = load_slot(p, row0, kbeg, sc + kPF * kWarps, c);
                if (MODE == MODE_MMA) {
                    uint32_t wa[16], wb[16];
                    dq_chunk(cur.p0, cur.z0, wa);
                    dq_chunk(cur.p1, cur.z1, wb);
                    const half2 s0 = scale_h2(cur.s0, p.scale_f16);
                    const half2 s1 = scale_h2(cur.s1, p.scale_f16);
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        wa[j] = h2_as_u32(__hmul2(u32_as_h2(wa[j]), s0));
                        wb[j] = h2_as_u32(__hmul2(u32_as_h2(wb[j]), s1));
                    }
#pragma unroll
                    for (int t = 0; t < NT; t++) {
                        const uint32_t xa = xs_base + (g + 8 * t) * p.xs_stride + sc * 256 + c * 16;
                        uint32_t xb[16];
#pragma unroll
                        for (int w = 0; w < 4; w++) {
                            const uint4 v = lds128(xa + w * 64);
                            xb[4 * w + 0] = v.x; xb[4 * w + 1] = v.y;
                            xb[4 * w + 2] = v.z; xb[4 * w + 3] = v.w;
                        }
#pragma unroll
                        for (int q = 0; q < 8; q++) {
                            const uint32_t a[4] = {wa[2 * q], wb[2 * q], wa[2 * q + 1], wb[2 * q + 1]};
                            mma16816(accm[t], a, xb[2 * q], xb[2 * q + 1]);
                        }
                    }
                } else if (ACT_F16) {
                    uint32_t wa[16], wb[16];
                    dq_chunk(cur.p0, cur.z0, wa);
                    dq_chunk(cur.p1, cur.z1, wb);
                    const float s0 = scale_f32(cur.s0, p.scale_f16);
                    const float s1 = scale_f32(cur.s1, p.scale_f16);
#pragma unroll
                    for (int m = 0; m < MP; m++) {
                        const uint32_t xa = xs_base + m * p.xs_stride + sc * 256 + c * 16;
                        uint32_t xb[16];
#pragma unroll
                        for (int w = 0; w < 4; w++) {
                            const uint4 v = lds128(xa + w * 64);
                            xb[4 * w + 0] = v.x; xb[4 * w + 1] = v.y;
                            xb[4 * w + 2] = v.z; xb[4 * w + 3] = v.w;
                        }
                        half2 a0 = __float2half2_rn(0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            a0 = __hfma2(u32_as_h2(wa[j]), u32_as_h2(xb[j]), a0);
                            a1 = __hfma2(u32_as_h2(wa[j + 1]), u32_as_h2(xb[j + 1]), a1);
                            b0 = __hfma2(u32_as_h2(wb[j]), u32_as_h2(xb[j]), b0);
                            b1 = __hfma2(u32_as_h2(wb[j + 1]), u32_as_h2(xb[j + 1]), b1);
                        }
                        const float2 fa0 = __half22float2(a0), fa1 = __half22float2(a1);
                        const float2 fb0 = __half22float2(b0), fb1 = __half22float2(b1);
                        accc[0][m] = fmaf(s0, (fa0.x + fa0.y) + (fa1.x + fa1.y), accc[0][m]);
                        accc[1][m] = fmaf(s1, (fb0.x + fb0.y) + (fb1.x + fb1.y), accc[1][m]);
                    }
                } else {
                    // fp32 activations: exact (q - zp) as fp32 via 2^23 + q
                    const float s0 = scale_f32(cur.s0, p.scale_f16);
                    const float s1 = scale_f32(cur.s1, p.scale_f16);
                    const float zb0 = 8388608.f + (float)cur.z0, zb1 = 8388608.f + (float)cur.z1;
                    const uint32_t w0[4] = {cur.p0.x, cur.p0.y, cur.p0.z, cur.p0.w};
                    const uint32_t w1[4] = {cur.p1.x, cur.p1.y, cur.p1.z, cur.p1.w};
                    float fa[32], fb[32];
#pragma unroll
                    for (int e = 0; e < 32; e++) {
                        const uint32_t na = (w0[e >> 3] >> (4 * (e & 7))) & 15u;
                        const uint32_t nb = (w1[e >> 3] >> (4 * (e & 7))) & 15u;
                        fa[e] = __uint_as_float(0x4B000000u | na) - zb0;
                        fb[e] = __uint_as_float(0x4B000000u | nb) - zb1;
                    }
#pragma unroll
                    for (int m = 0; m < MP; m++) {
                        const uint32_t xa = xs_base + m * p.xs_stride + sc * 512 + c * 16;
                        float pa = 0.f, pb = 0.f;
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const uint4 v = lds128(xa + j * 64);
                            const float xv[4] = {__uint_as_float(v.x), __uint_as_float(v.y),
                                                 __uint_as_float(v.z), __uint_as_float(v.w)};
#pragma unroll
                            for (int e = 0; e < 4; e++) {
                                pa = fmaf(xv[e], fa[4 * j + e], pa);
                                pb = fmaf(xv[e], fb[4 * j + e], pb);
                            }
                        }
                        accc[0][m] = fmaf(s0, pa, accc[0][m]);
                        accc[1][m] = fmaf(s1, pb, accc[1][m]);
                    }
                }
            }
        }
    }

    // ---- reduce: lanes -> warp partials in shared memory
    if (MODE == MODE_MMA) {
#pragma unroll
        for (int t = 0; t < NT; t++) {
            const int m0 = 8 * t + 2 * c;
            red[(warp * kRows + g) * MP + m0] = accm[t][0];
            red[(warp * kRows + g) * MP + m0 + 1] = accm[t][1];
            red[(warp * kRows + g + 8) * MP + m0] = accm[t][2];
            red[(warp * kRows + g + 8) * MP + m0 + 1] = accm[t][3];
        }
    } else {
#pragma unroll
        for (int r = 0; r < 2; r++)
#pragma unroll
            for (int m = 0; m < MP; m++) {
                float v = accc[r][m];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                if (c == 0)
                    red[(warp * kRows + g + 8 * r) * MP + m] = v;
            }
    }
    __syncthreads();
    for (int i = tid; i < kRows * MP; i += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; w++)
            v += red[w * kRows * MP + i];
        part[i] = v;
    }

    // ---- reduce across the cluster through distributed shared memory
    if (p.S > 1)
        cluster_sync();
    if (rank == 0) {
        for (int i = tid; i < kRows * MP; i += kThreads) {
            const int r = i / MP, m = i - r * MP;
            const int n = tile * kRows + r;
            if (m >= p.M || n >= p.N)
                continue;
            float v = part[i];
            for (int q = 1; q < p.S; q++)
                v += ld_dsmem_f32(part + i, (uint32_t)q);
            if (ACT_F16)
                reinterpret_cast<__half *>(p.Y)[(int64_t)m * p.N + n] = __float2half_rn(v);
            else
                reinterpret_cast<float *>(p.Y)[(int64_t)m * p.N + n] = v;
        }
    }
    if (p.S > 1)
        cluster_sync();   // keep every CTA's shared memory alive until rank 0 has read it
}

template <int MODE, bool ACT_F16, int MP>
int launch_one(const Params &p, int grid, size_t smem, unsigned flags, cudaStream_t s) {
    auto fn = gemv_kernel<MODE, ACT_F16, MP>;
    static int configured = 0;   // largest dynamic shared memory opted into so far
    if ((int)smem > 48 * 1024 && (int)smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured = (int)smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (p.S > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)p.S;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        na++;
    }
    if (flags & MNB_FLAG_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        na++;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

int sm_count() {
    static int count = 0;
    if (count == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || count <= 0)
            count = 148;
    }
    return count;
}

}  // namespace

// Which inner product serves fp16 activations at M = 1 and 2: MMA by default.
static int g_gemv_f16_cc_max_m = 0;

int launch_gemv(const void *X, int act_f16, const uint8_t *packed, const void *scales,
                int scale_f16, const uint8_t *zp, void *Y, int M, int N, int K, int bs,
                unsigned flags, cudaStream_t s) {
    const int mode = (act_f16 && M > g_gemv_f16_cc_max_m) ? MODE_MMA : MODE_CC;
    int MP;
    if (mode == MODE_MMA)
        MP = (M <= 8) ? 8 : 16;
    else
        MP = (M <= 1) ? 1 : (M <= 2) ? 2 : (M <= 4) ? 4 : (M <= 8) ? 8 : 16;
    const int esz = act_f16 ? 2 : 4;

    Params p;
    p.X = X; p.packed = packed; p.scales = scales; p.zp = zp; p.Y = Y;
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.scale_f16 = scale_f16;

    const int tiles = (N + kRows - 1) / kRows;
    const int want = 2 * sm_count();
    int S = (want + tiles - 1) / tiles;
    const int s_k = K / 512 > 0 ? K / 512 : 1;   // keep >= 4 super-chunks per split
    if (S > s_k) S = s_k;
    if (S > kMaxCluster) S = kMaxCluster;
    if (S < 1) S = 1;
    const size_t kSmemCap = 96 * 1024;
    size_t smem = 0;
    for (;; S++) {
        const int ks = ((K + S - 1) / S + kSuper - 1) / kSuper * kSuper;
        const int nsc = ks / kSuper;
        const int xs_stride = nsc * kSuper * esz + 64;
        smem = (size_t)MP * xs_stride + (size_t)(kWarps + 1) * kRows * MP * 4;
        p.S = S; p.ks = ks; p.nsc = nsc; p.xs_stride = xs_stride;
        if (smem <= kSmemCap || S >= kMaxCluster)
            break;
    }
    if (smem > 200 * 1024)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: K=%d too large for M=%d", K, M);
    if ((int64_t)tiles * p.S > 0x7fffffff)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: N too large");
    const int grid = tiles * p.S;

    if (mode == MODE_MMA) {
        if (MP == 8) return launch_one<MODE_MMA, true, 8>(p, grid, smem, flags, s);
        return launch_one<MODE_MMA, true, 16>(p, grid, smem, flags, s);
    }
    if (act_f16) {
        if (MP == 1) return launch_one<MODE_CC, true, 1>(p, grid, smem, flags, s);
        return launch_one<MODE_CC, true, 2>(p, grid, smem, flags, s);
    }
    switch (MP) {
        case 1: return launch_one<MODE_CC, false, 1>(p, grid, smem, flags, s);
        case 2: return launch_one<MODE_CC, false, 2>(p, grid, smem, flags, s);
        case 4: return launch_one<MODE_CC, false, 4>(p, grid, smem, flags, s);
        case 8: return launch_one<MODE_CC, false, 8>(p, grid, smem, flags, s);
        default: return launch_one<MODE_CC, false, 16>(p, grid, smem, flags, s);
    }
}

}  // namespace mnb

// Tuning hook: fp16 GEMVs with M <= max_m use the CUDA-core inner product
// (0 = always the tensor-core one; at most 2).  Not part of the stable ABI.
extern "C" MNB_API int mnb_tune_gemv_f16_cc_max_m(int max_m) {
    if (max_m < 0 || max_m > 2)
        return MNB_ERR_INVALID_ARG;
    mnb::g_gemv_f16_cc_max_m = max_m;
    return MNB_OK;
}
