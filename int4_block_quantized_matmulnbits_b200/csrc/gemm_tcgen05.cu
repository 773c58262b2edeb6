// gemm_tcgen05.cu -- prefill-shaped MatMulNBits on the 5th-generation tensor
// cores: Y[M][N] = X[M][K] . dequant(W)^T with fp16 X and Y (the full-length
// prefill of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", "What's in this repo":
// decoder_prefill_int4, and decoder_init of "Qwen3-ASR-0.6B -- ONNX for the
// browser", "Graph contracts").
//
// A dense contraction, so it runs on tcgen05.mma (kind::f16, fp32 accumulation
// in tensor memory).  Weight rows are the MMA's M (128 per CTA) and tokens its N
// (BN <= 256), so ragged token counts only pad N.
//
// Per CTA, a K loop over 64-wide stages in a ring of shared-memory buffers:
//   warp 0     TMA producer: X tile [BN x 64] fp16, 128-byte swizzle.  Also
//              allocates / frees the tensor-memory accumulator.
//   warp 1     MMA issuer: one thread issues 4 x tcgen05.mma (K = 16 each) per
//              stage and commits to the stage's "empty" barrier.
//   warps 2-5  dequant producers, one weight row per thread: 32 packed bytes
//              -> 64 fp16 = fp16_rn((q - zp) * scale), written in the
//              128-byte-swizzled K-major layout the MMA descriptor reads, then
//              fence.proxy.async + mbarrier arrive.  Their global loads run a
//              few stages ahead in a register ring.  After the K loop the same
//              warps are the epilogue: tcgen05.ld of their 32 TMEM lanes,
//              fp16 conversion, coalesced stores of Y.
// Every mbarrier wait is bounded in time: past the limit the kernel records
// the failure in a device status word, drains what it issued, frees tensor
// memory and exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace mnb {

__device__ unsigned g_mnb_status = 0;

namespace {

constexpr int kThreads = 192;   // 6 warps
constexpr int kBM = 128;        // weight rows per CTA
constexpr int kBK = 64;         // k per stage (128 bytes of fp16 = one swizzle row)
constexpr int kWRing = 3;       // dequant loads in flight per thread
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

struct GemmParams {
    const uint8_t *packed;
    const void *scales;
    const uint8_t *zp;
    __half *Y;
    int M, N, K;
    int bs_shift, nb, zpb, scale_f16;
    int BN;        // tokens per CTA (multiple of 16, <= 256)
    int stages;    // shared-memory ring depth
    int tmem_cols; // power of two >= BN
};

// ---- mbarrier / TMA / tcgen05 wrappers -------------------------------------

// Waits for the phase with the given parity; false after the time limit or,
// unless `drain`, as soon as another role has given up (*abort set).  Drain
// waits (used to let issued copies and MMAs land before exit) only stop at the
// time limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          bool drain = false) {
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255) == 0) {
            if (*abort && !drain)
                return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicOr(&g_mnb_status, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
            tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t v[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
        "[%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- dequant of one stage of one weight row --------------------------------

struct WSlot {
    uint4 p0, p1;       // k 0..31 and 32..63 of the stage
    uint32_t s0, s1;    // fp16 bits of the scales of the (up to) two blocks
    uint32_t z0, z1;    // zero points
};

__device__ __forceinline__ WSlot load_wslot(const GemmParams &p, int n, int it, int nk) {
    WSlot w;
    w.p0 = w.p1 = make_uint4(0, 0, 0, 0);
    w.s0 = w.s1 = 0;
    w.z0 = w.z1 = 8;
    if (it >= nk)
        return w;
    const int k0 = it * kBK;
    const uint8_t *row = p.packed + (int64_t)n * (p.K / 2) + k0 / 2;
    w.p0 = ldg_stream_v4(row);
    w.p1 = ldg_stream_v4(row + 16);
    const int b0 = k0 >> (5 + p.bs_shift);
    const int b1 = (k0 + 32) >> (5 + p.bs_shift);
    if (p.scale_f16) {
        const unsigned short *s = reinterpret_cast<const unsigned short *>(p.scales) + (int64_t)n * p.nb;
        w.s0 = __ldg(s + b0);
        w.s1 = __ldg(s + b1);
    } else {
        // fp32 scales: the tensor cores take fp16 operands, so round the scale once here
        const float *s = reinterpret_cast<const float *>(p.scales) + (int64_t)n * p.nb;
        w.s0 = __half_as_ushort(__float2half_rn(__ldg(s + b0)));
        w.s1 = __half_as_ushort(__float2half_rn(__ldg(s + b1)));
    }
    if (p.zp) {
        const uint8_t *z = p.zp + (int64_t)n * p.zpb;
        const uint32_t zb0 = __ldg(z + (b0 >> 1)), zb1 = __ldg(z + (b1 >> 1));
        w.z0 = (b0 & 1) ? (zb0 >> 4) : (zb0 & 15);
        w.z1 = (b1 & 1) ? (zb1 >> 4) : (zb1 & 15);
    }
    return w;
}

// 32 nibbles -> 32 fp16 = fp16_rn((q - zp) * s) in natural k order, written as
// four 16-byte chunks (k 8j..8j+7) of the swizzled row.
__device__ __forceinline__ void dq_store_half_row(const uint4 &p, uint32_t s16, uint32_t z, uint32_t row_addr,
                                                  int r7, int j0) {
    const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    const half2 s2 = u32_as_h2(s16 | (s16 << 16));
    const uint32_t Z = 0x64006400u | (z * 0x00010001u);
    const uint32_t Zhi = 0xD400D400u + (z * 0x00100010u);
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t w = words[i];
        const uint32_t w8 = w >> 8;
        // (e0,e4) (e1,e5) (e2,e6) (e3,e7) as exact q - zp, then times the scale
        const half2 P0 = __hmul2(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s2);
        const half2 P1 = __hmul2(__hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth,
                                         u32_as_h2(Zhi)), s2);
        const half2 P2 = __hmul2(__hsub2(u32_as_h2(lop3_and_or(w8, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s2);
        const half2 P3 = __hmul2(__hfma2(u32_as_h2(lop3_and_or(w8, 0x00F000F0u, 0x64006400u)), sixteenth,
                                         u32_as_h2(Zhi)), s2);
        const uint32_t a = h2_as_u32(P0), b = h2_as_u32(P1), c = h2_as_u32(P2), d = h2_as_u32(P3);
        uint4 o;
        o.x = __byte_perm(a, b, 0x5410);   // (e0, e1)
        o.y = __byte_perm(c, d, 0x5410);   // (e2, e3)
        o.z = __byte_perm(a, b, 0x7632);   // (e4, e5)
        o.w = __byte_perm(c, d, 0x7632);   // (e6, e7)
        const int j = j0 + i;
        const uint32_t dst = row_addr + (uint32_t)(((j ^ r7) & 7) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w)
                     : "memory");
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap xmap, const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int S = p.stages;
    const int BN = p.BN;
    const int n_tile = blockIdx.x;          // weight-row tile
    const int m_tile = blockIdx.y;          // token tile
    const int nk = p.K / kBK;

    // layout: [stages][W 16 KB][X BN*128 B] (1024-aligned), then barriers
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *base_ptr = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t w_bytes = kBM * 128;
    const uint32_t x_bytes = (uint32_t)BN * 128;
    const uint32_t stage_bytes = w_bytes + x_bytes;
    const uint32_t bar_base = base + (uint32_t)S * stage_bytes;
    // barriers: full_x[S], full_w[S], empty[S], acc_full; then tmem addr, abort flag
    auto full_x = [&](int s) { return bar_base + 8u * (uint32_t)s; };
    auto full_w = [&](int s) { return bar_base + 8u * (uint32_t)(S + s); };
    auto empty = [&](int s) { return bar_base + 8u * (uint32_t)(2 * S + s); };
    const uint32_t acc_full = bar_base + 8u * (uint32_t)(3 * S);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (size_t)S * stage_bytes + 8 * (3 * S + 1));
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(full_x(s), 1);
            mbar_init(full_w(s), 128);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full, 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer of X tiles
            pdl_wait();
            int issued = 0;
            for (int it = 0; it < nk; it++) {
                const int s = it % S;
                if (it >= S && !mbar_wait(empty(s), ((it / S) - 1) & 1, abort))
                    break;
                mbar_expect_tx(full_x(s), x_bytes);
                tma_load_2d(base + (uint32_t)s * stage_bytes + w_bytes, &xmap, full_x(s), it * kBK, m_tile * BN);
                issued = it + 1;
            }
            if (*abort) {
                // drain: every issued load must land before the CTA exits
                for (int it = (issued > S ? issued - S : 0); it < issued; it++)
                    mbar_wait(full_x(it % S), (it / S) & 1, abort, true);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
            for (int it = 0; it < nk; it++) {
                const int s = it % S;
                const uint32_t par = (it / S) & 1;
                if (!mbar_wait(full_x(s), par, abort) || !mbar_wait(full_w(s), par, abort))
                    break;
                tc_fence_after();
                const uint32_t wa = base + (uint32_t)s * stage_bytes;
                const uint32_t xa = wa + w_bytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; kk++)
                    tc_mma_f16(tmem, sw128_desc(wa + kk * 32), sw128_desc(xa + kk * 32), idesc,
                               (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(empty(s));
            }
            tc_commit(acc_full);   // fires once every MMA issued above has completed
        }
    } else {
        // ---------------- dequant producers (one weight row each), then epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;             // row within the tile
        const int n = n_tile * kBM + r;
        const int r7 = r & 7;
        WSlot ring[kWRing];
#pragma unroll
        for (int i = 0; i < kWRing; i++)
            ring[i] = load_wslot(p, n, i, nk);
        bool ok = true;
        for (int base_it = 0; base_it < nk && ok; base_it += kWRing) {
#pragma unroll
            for (int i = 0; i < kWRing; i++) {
                const int it = base_it + i;
                if (it < nk && ok) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait(empty(s), ((it / S) - 1) & 1, abort)) {
                        ok = false;
                    } else {
                        const WSlot cur = ring[i];
                        ring[i] = load_wslot(p, n, it + kWRing, nk);
                        const uint32_t row_addr = base + (uint32_t)s * stage_bytes + (uint32_t)r * 128;
                        dq_store_half_row(cur.p0, cur.s0, cur.z0, row_addr, r7, 0);
                        dq_store_half_row(cur.p1, cur.s1, cur.z1, row_addr, r7, 4);
                        fence_proxy_async_smem();
                        mbar_arrive(full_w(s));
                    }
                }
            }
        }
        // ---------------- epilogue: TMEM -> registers -> Y
        if (mbar_wait(acc_full, 0, abort)) {
            tc_fence_after();
            pdl_wait();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
            const int m0 = m_tile * BN;
            for (int col = 0; col < BN; col += 16) {
                uint32_t v[16];
                tc_ld16(taddr + (uint32_t)col, v);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int m = m0 + col + j;
                    if (m < p.M)
                        p.Y[(int64_t)m * p.N + n] = __float2half_rn(__uint_as_float(v[j]));
                }
            }
        }
    }

    // ---------------- teardown
    if (*abort && warp == 1 && lane == 0)
        mbar_wait(acc_full, 0, abort, true);   // let the issued MMAs finish before freeing TMEM
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

// ---- host side ----------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

int launch_gemm(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s) {
    EncodeTiledFn encode = get_encode_fn();
    if (!encode)
        return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled unavailable");

    // token tiling: as few tiles of <= 256 as possible, evenly sized
    int mt = (M + 255) / 256;
    int BN = ((M + mt - 1) / mt + 15) / 16 * 16;
    const int n_tiles = N / kBM;
    int sms = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    // narrower token tiles when the grid would leave most SMs idle
    while (BN > 64 && (int64_t)n_tiles * mt * 2 <= sms) {
        mt = (M + BN / 2 - 1) / (BN / 2);
        BN = ((M + mt - 1) / mt + 15) / 16 * 16;
    }
    if (mt > 65535)
        return fail(MNB_ERR_SHAPE, "mnb_gemm: M too large");

    GemmParams p;
    p.packed = packed;
    p.scales = scales;
    p.zp = zp;
    p.Y = reinterpret_cast<__half *>(Y);
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.scale_f16 = scale_f16;
    p.BN = BN;
    p.tmem_cols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
    const int stage_bytes = kBM * 128 + BN * 128;
    const int budget = 200 * 1024;
    int stages = budget / stage_bytes;
    if (stages > 8) stages = 8;
    if (stages < 2) stages = 2;
    p.stages = stages;
    const size_t smem = 1024 + (size_t)stages * stage_bytes + 8 * (3 * stages + 1) + 16;

    CUtensorMap xmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(X), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS)
        return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled failed (%d)", (int)cr);

    static int configured = 0;
    if ((int)smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemm: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured = (int)smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_tiles, (unsigned)mt, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (flags & MNB_FLAG_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        na++;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel, xmap, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemm: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

int read_device_status(unsigned *out, int clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_mnb_status, sizeof(unsigned));
    if (e == cudaSuccess) {
        const int rc = read_gemv_status(out, clear);
        if (rc)
            return rc;
    }
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_mnb_status, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_device_status: %s", cudaGetErrorString(e));
    return MNB_OK;
}

}  // namespace mnb
