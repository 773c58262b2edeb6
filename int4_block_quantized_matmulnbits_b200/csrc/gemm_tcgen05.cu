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
// Per CTA, a K loop over 64-wide stages fed by three shared-memory rings (packed
// weights 8 deep, X tiles up to 8 deep, fp16 weight tiles 4 deep), so the long
// DRAM latency of the weight stream is covered without holding X or fp16 space:
//   warp 0      TMA producer of the packed weight tile (128 rows x 32 bytes) of
//               every stage; it never waits for the previous kernel, whose
//               output the weights do not depend on.  Also allocates / frees the
//               tensor-memory accumulator.
//   warp 2      TMA producer of the X tile [BN x 64] fp16 (128-byte swizzle),
//               after griddepcontrol.wait.
//   warp 1      MMA issuer: one thread issues 4 x tcgen05.mma (K = 16 each) per
//               stage and commits to the X and fp16-weight "empty" barriers.
//   warps 3-18  dequant, in two groups of eight that take alternate stages (two
//               stages are unpacked at once): two threads per weight row, 32 k
//               each per stage: 16 packed bytes from shared memory -> 32 fp16 =
//               fp16_rn((q - zp) * scale), written in the 128-byte-swizzled
//               K-major layout the MMA descriptor reads, then fence.proxy.async,
//               __syncwarp and one mbarrier arrival per warp.
//               Scales and zero points run a few stages ahead in registers.
//               After the K loop the same warps are the epilogue: tcgen05.ld of
//               their 32 TMEM lanes, fp16 conversion, stores of Y.
// When rows x token tiles cannot occupy the SMs, K is split over a cluster of S
// CTAs; each keeps its partial sum in its own tensor memory.  Every rank owns
// a contiguous slice of the token columns: the others write their parts of it
// straight from tensor memory into its shared memory (distributed shared
// memory stores), and it adds them to its own in rank order and stores the
// slice by TMA (no global scratch).
// Every mbarrier wait is bounded in time: past the limit the kernel records
// the failure in a device status word, drains what it issued, frees tensor
// memory and exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "mnb_tune.h"

namespace mnb {

__device__ unsigned g_mnb_status = 0;

namespace {

constexpr int kDqWarps = 16;
constexpr int kThreads = 96 + kDqWarps * 32;   // 2 TMA producers, MMA, 16 dequant warps
constexpr int kBM = 128;                       // weight rows per CTA
constexpr int kBK = 64;                        // k per stage (128 bytes of fp16 = one swizzle row)
constexpr int kWBytes = kBM * 128;             // fp16 weight tile per stage
constexpr int kPBytes = kBM * 32;              // packed weight tile per stage
constexpr int kPR = 4;                         // stages of scales / zero points prefetched
constexpr int kWS = 4;                         // fp16 weight tiles in the ring
constexpr int kPS = 8;                         // packed weight tiles in flight
constexpr int kMaxCluster = 8;
constexpr uint32_t kChunkBytes = kBM * 16 * 4;   // one 16-column chunk of fp32 partial sums
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

struct GemmParams {
    const void *scales;
    const uint8_t *zp;
    __half *Y;
    int M, N, K;
    int bs_shift, nb, zpb;
    int BN;        // tokens per CTA (multiple of 16, <= 256)
    int xstages;   // depth of the X ring
    int tmem_cols; // power of two >= BN
    int S;         // CTAs per cluster along K
    int kslice;    // k per cluster rank (multiple of kBK)
};

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

// mbar_wait by a whole warp with a warp-uniform result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

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




// Address of the same shared-memory location in cluster rank `rank`.
__device__ __forceinline__ uint32_t map_cluster(uint32_t local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    return remote;
}

// Scale (fp16 bits) and zero point of one thread's 32-k half of a stage (one
// block of 32, or half a block of 64).
struct SZ {
    uint32_t s, z;
};

__device__ __forceinline__ SZ load_sz(const GemmParams &p, int n, int k) {
    SZ r;
    r.s = 0;
    r.z = 8;
    if (k >= p.K)
        return r;
    const int b = k >> (5 + p.bs_shift);
    r.s = __ldg(reinterpret_cast<const unsigned short *>(p.scales) + (int64_t)n * p.nb + b);   // fp16 scales only
    if (p.zp) {
        const uint32_t zb = __ldg(p.zp + (int64_t)n * p.zpb + (b >> 1));
        r.z = (b & 1) ? (zb >> 4) : (zb & 15u);
    }
    return r;
}

// 8 packed bytes (16 k of one row) -> 16 fp16 = fp16_rn((q - zp) * s) in natural
// k order, written as two 16-byte chunks (k 8j..8j+7, j = j0, j0+1) of the
// row's 128-byte swizzled line.
__device__ __forceinline__ void dq_store(const uint2 &v, uint32_t s16, uint32_t z, uint32_t row_addr, int r7,
                                         int j0) {
    const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    const half2 s2 = u32_as_h2(s16 | (s16 << 16));
    const uint32_t Z = 0x64006400u | (z * 0x00010001u);      // 1024 + zp
    const uint32_t Zhi = 0xD400D400u + (z * 0x00100010u);    // -(64 + zp)
    const uint32_t words[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 2; i++) {
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
        const uint32_t dst = row_addr + (uint32_t)((((j0 + i) ^ r7) & 7) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w)
                     : "memory");
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                const __grid_constant__ CUtensorMap ymap, const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int WS = kWS, PS = kPS, XS = p.xstages;
    const int BN = p.BN;
    const int rank = (p.S > 1) ? (int)cluster_ctarank() : 0;
    const int n_tile = blockIdx.x / p.S;    // weight-row tile
    const int m_tile = blockIdx.y;          // token tile
    const int kbeg = rank * p.kslice;
    const int kend = min(p.K, kbeg + p.kslice);
    const int nk = (kend > kbeg) ? (kend - kbeg) / kBK : 0;

    // layout (1024-aligned): W16 ring [WS][16 KB] | X ring [XS][BN*128 B] |
    // packed ring [PS][4 KB] | barriers
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *base_ptr = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t x_bytes = (uint32_t)BN * 128;
    const uint32_t x_base = base + (uint32_t)WS * kWBytes;
    const uint32_t p_base = x_base + (uint32_t)XS * x_bytes;
    auto w_addr = [&](int i) { return base + (uint32_t)(i % WS) * kWBytes; };
    auto x_addr = [&](int i) { return x_base + (uint32_t)(i % XS) * x_bytes; };
    auto p_off = [&](int i) { return (p_base - base) + (uint32_t)(i % PS) * kPBytes; };
    const uint32_t bars = p_base + (uint32_t)PS * kPBytes;
    auto pfull = [&](int i) { return bars + 8u * (uint32_t)(i % PS); };
    auto pempty = [&](int i) { return bars + 8u * (uint32_t)(PS + i % PS); };
    auto wfull = [&](int i) { return bars + 8u * (uint32_t)(2 * PS + i % WS); };
    auto wempty = [&](int i) { return bars + 8u * (uint32_t)(2 * PS + WS + i % WS); };
    auto xfull = [&](int i) { return bars + 8u * (uint32_t)(2 * PS + 2 * WS + i % XS); };
    auto xempty = [&](int i) { return bars + 8u * (uint32_t)(2 * PS + 2 * WS + XS + i % XS); };
    const uint32_t acc_full = bars + 8u * (uint32_t)(2 * PS + 2 * WS + 2 * XS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (acc_full + 16 - base));
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    if (tid == 0) {
        for (int i = 0; i < PS; i++) {
            mbar_init(pfull(i), 1);
            mbar_init(pempty(i), kDqWarps / 2);   // the 8 warps of the group that unpacks it
        }
        for (int i = 0; i < WS; i++) {
            mbar_init(wfull(i), kDqWarps / 2);
            mbar_init(wempty(i), 1);
        }
        for (int i = 0; i < XS; i++) {
            mbar_init(xfull(i), 1);
            mbar_init(xempty(i), 1);
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

    // The producer and MMA warps run their loops with all 32 lanes (lane 0
    // issues); a warp left diverged for the whole K loop runs far slower.
    if (warp == 0) {
        // ---------------- TMA producer of packed weights (independent of the
        // previous kernel: no griddepcontrol.wait)
        int issued = 0;
        for (int i = 0; i < nk; i++) {
            if (i >= PS && !warp_wait(pempty(i), ((i / PS) - 1) & 1, abort))
                break;
            if (lane == 0) {
                mbar_expect_tx(pfull(i), kPBytes);
                tma_load_2d(base + p_off(i), &wmap, pfull(i), (kbeg + i * kBK) / 2, n_tile * kBM);
            }
            __syncwarp();
            issued = i + 1;
        }
        if (*abort)
            for (int i = (issued > PS ? issued - PS : 0); i < issued; i++)
                mbar_wait(pfull(i), (i / PS) & 1, abort, true);
    } else if (warp == 2) {
        // ---------------- TMA producer of X tiles
        pdl_wait();
        int issued = 0;
        for (int i = 0; i < nk; i++) {
            if (i >= XS && !warp_wait(xempty(i), ((i / XS) - 1) & 1, abort))
                break;
            if (lane == 0) {
                mbar_expect_tx(xfull(i), x_bytes);
                tma_load_2d(x_addr(i), &xmap, xfull(i), kbeg + i * kBK, m_tile * BN);
            }
            __syncwarp();
            issued = i + 1;
        }
        if (*abort)
            for (int i = (issued > XS ? issued - XS : 0); i < issued; i++)
                mbar_wait(xfull(i), (i / XS) & 1, abort, true);
    } else if (warp == 1) {
        // ---------------- MMA issuer
        const uint32_t idesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
        for (int i = 0; i < nk; i++) {
            if (!warp_wait(xfull(i), (i / XS) & 1, abort) || !warp_wait(wfull(i), (i / WS) & 1, abort))
                break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < kBK / 16; kk++)
                    tc_mma_f16(tmem, sw128_desc(w_addr(i) + kk * 32), sw128_desc(x_addr(i) + kk * 32), idesc,
                               (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(xempty(i));
                tc_commit(wempty(i));
            }
            __syncwarp();
        }
        if (lane == 0)
            tc_commit(acc_full);   // fires once every MMA issued above has completed
        __syncwarp();
    } else {
        // ---------------- dequant: two groups of 8 warps take alternate stages, so
        // two stages are being unpacked at once; in a group, thread = (row r,
        // half hh of the stage's 64 k): 16 packed bytes -> 32 fp16
        const int dt = tid - 96;
        const int dgrp = dt >> 8, t = dt & 255;
        const int r = t >> 1, hh = t & 1;
        const int n = n_tile * kBM + r;
        const int r7 = r & 7;
        SZ ring[kPR];
#pragma unroll
        for (int i = 0; i < kPR; i++) {
            const int it = dgrp + 2 * i;
            ring[i] = (it < nk) ? load_sz(p, n, kbeg + it * kBK + hh * 32) : SZ{0u, 8u};
        }
        bool ok = true;
        for (int base_j = 0; dgrp + 2 * base_j < nk && ok; base_j += kPR) {
#pragma unroll
            for (int i = 0; i < kPR; i++) {
                const int it = dgrp + 2 * (base_j + i);
                if (it < nk && ok) {
                    // warp-uniform outcome, so the warp stays converged for __syncwarp
                    ok = __all_sync(0xffffffffu, mbar_wait(pfull(it), (it / PS) & 1, abort) &&
                                                     (it < WS || mbar_wait(wempty(it), ((it / WS) - 1) & 1, abort)));
                    if (ok) {
                        const SZ cur = ring[i];
                        const int nxt = it + 2 * kPR;
                        if (nxt < nk)
                            ring[i] = load_sz(p, n, kbeg + nxt * kBK + hh * 32);
                        const uint4 v = *reinterpret_cast<const uint4 *>(base_ptr + p_off(it) + r * 32 + hh * 16);
                        // one arrival per warp: hundreds of arrivals on one mbarrier serialise
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(pempty(it));   // the warp's packed bytes are in registers now
                        const uint32_t row_addr = w_addr(it) + (uint32_t)r * 128;
                        dq_store(make_uint2(v.x, v.y), cur.s, cur.z, row_addr, r7, hh * 4);
                        dq_store(make_uint2(v.z, v.w), cur.s, cur.z, row_addr, r7, hh * 4 + 2);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(wfull(it));
                    }
                }
            }
        }

        // ---------------- epilogue: TMEM -> registers -> (cluster reduction) -> Y
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int grp = (warp - 3) >> 2;         // 0..3: this warp's share of the column chunks
        const int row = q * 32 + lane;
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
        const int m0 = m_tile * BN;
        const int nchunk = BN / 16;
        const bool have = mbar_wait(acc_full, 0, abort) && nk > 0;
        tc_fence_after();
        pdl_wait();
        if (p.S == 1) {
            // the tile goes through shared memory (the idle fp16 weight ring) as
            // [BN tokens][128 rows] fp16 and leaves in one TMA store; two 16-column
            // chunks per tensor-memory load round trip
            __half *stage = reinterpret_cast<__half *>(base_ptr);
            for (int c16 = grp; c16 < nchunk; c16 += 8) {
                const bool two = c16 + 4 < nchunk;
                uint32_t v[2][16];
                if (have) {
                    tc_ld16(taddr + (uint32_t)(c16 * 16), v[0]);
                    if (two)
                        tc_ld16(taddr + (uint32_t)((c16 + 4) * 16), v[1]);
                    tc_wait_ld();
                }
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    if (h == 1 && !two)
                        break;
                    const int col = (c16 + 4 * h) * 16;
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        stage[(col + j) * kBM + row] = __float2half_rn(have ? __uint_as_float(v[h][j]) : 0.f);
                }
            }
            fence_proxy_async_smem();   // the TMA store reads what the generic stores wrote
            asm volatile("bar.sync 1, %0;" ::"n"(kDqWarps * 32) : "memory");
            if (warp == 3 && lane == 0 && have) {
                asm volatile(
                    "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(&ymap),
                    "r"(n_tile * kBM), "r"(m0), "r"(smem_u32(stage))
                    : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // written before the CTA leaves
            }
        } else {
            // K split over the cluster.  Chunk c (16 token columns) belongs to
            // rank c / per: contiguous ranges.  Once every rank's K loop is over
            // (its rings are free), each rank writes the chunks it does not own
            // straight from tensor memory into the owner's receive area
            // (distributed shared memory stores; [sender slot][owned chunk]
            // [row][16] fp32).  After a second cluster barrier each owner adds
            // to its own sums, read again from tensor memory, the received
            // parts in rank order, and its chunks leave through shared memory
            // and TMA stores.
            const int per = (nchunk + p.S - 1) / p.S;
            float *recv = reinterpret_cast<float *>(base_ptr);   // reuses the ring buffers
            __half *stage = reinterpret_cast<__half *>(recv + (size_t)(p.S - 1) * per * kBM * 16);   // [per][16][128]
            cluster_sync();   // every rank is past its K loop: its shared memory may be written
            for (int c16 = grp; c16 < nchunk; c16 += 4) {
                const int owner = c16 / per;
                if (owner == rank)
                    continue;
                uint32_t v[16];
                if (have) {
                    tc_ld16(taddr + (uint32_t)(c16 * 16), v);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        v[j] = 0u;
                }
                const int slot = rank - (rank > owner ? 1 : 0);   // senders in rank order
                const uint32_t dst = map_cluster(
                    smem_u32(recv + (((size_t)slot * per + (c16 - owner * per)) * kBM + row) * 16), (uint32_t)owner);
#pragma unroll
                for (int i = 0; i < 4; i++)
                    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16u * i),
                                 "r"(v[4 * i]), "r"(v[4 * i + 1]), "r"(v[4 * i + 2]), "r"(v[4 * i + 3])
                                 : "memory");
            }
            cluster_sync();   // every part has landed
            const int c_lo = rank * per, c_hi = min(nchunk, c_lo + per);
            for (int c16 = c_lo + grp; c16 < c_hi; c16 += 4) {
                uint32_t v[16];
                if (have) {
                    tc_ld16(taddr + (uint32_t)(c16 * 16), v);
                    tc_wait_ld();
                }
                float f[16];
#pragma unroll
                for (int j = 0; j < 16; j++)
                    f[j] = have ? __uint_as_float(v[j]) : 0.f;
                for (int sl = 0; sl < p.S - 1; sl++) {
                    const float4 *in = reinterpret_cast<const float4 *>(recv + (((size_t)sl * per + (c16 - c_lo)) * kBM + row) * 16);
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const float4 o = in[j];
                        f[4 * j] += o.x; f[4 * j + 1] += o.y; f[4 * j + 2] += o.z; f[4 * j + 3] += o.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < 16; j++)
                    stage[((c16 - c_lo) * 16 + j) * kBM + row] = __float2half_rn(f[j]);
            }
            fence_proxy_async_smem();   // the TMA stores read what the generic stores wrote
            asm volatile("bar.sync 1, %0;" ::"n"(kDqWarps * 32) : "memory");
            if (warp == 3 && lane == 0 && have) {
                for (int c16 = c_lo; c16 < c_hi && m0 + c16 * 16 < p.M; c16++)   // no box wholly past M
                    asm volatile(
                        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(&ymap),
                        "r"(n_tile * kBM), "r"(m0 + c16 * 16), "r"(smem_u32(stage + (size_t)(c16 - c_lo) * 16 * kBM))
                        : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // written before the CTA leaves
            }
        }
    }
    if (p.S > 1 && warp < 3) {
        // the producer and MMA warps take part in the epilogue's cluster barriers
        cluster_sync();
        cluster_sync();
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

}  // namespace

// Tile policy knobs (tuning hooks, see mnb_tune_gemm below).
static int g_gemm_min_bn = 128;      // smallest token tile the grid heuristic may pick
static int g_gemm_max_bn = 256;      // largest token tile
// at most 4 CTAs per cluster: 8-CTA clusters of ~200 KB each wait for 8 free
// SMs of one GPC and measured up to 2x slower, never faster
static int g_gemm_max_split = 4;

int launch_gemm(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s) {
    EncodeTiledFn encode = tensor_map_encoder();
    if (!encode)
        return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled unavailable");
    const int sms = device_sm_count();

    // token tiling: as few tiles of <= 256 as possible, evenly sized; narrower
    // tiles (down to g_gemm_min_bn) while the grid would leave half the SMs idle
    int mt = (M + g_gemm_max_bn - 1) / g_gemm_max_bn;
    int BN = ((M + mt - 1) / mt + 15) / 16 * 16;
    const int n_tiles = N / kBM;
    while (BN > g_gemm_min_bn && BN > 16 && (int64_t)n_tiles * mt * 4 <= sms) {
        mt = (M + BN / 2 - 1) / (BN / 2);
        BN = ((M + mt - 1) / mt + 15) / 16 * 16;
    }
    if (mt > 65535)
        return fail(MNB_ERR_SHAPE, "mnb_gemm: M too large");
    // split K over a cluster when the tiles still leave most SMs idle
    const int nk_all = K / kBK;
    int S = 1;
    while (S * 2 <= g_gemm_max_split && (int64_t)n_tiles * mt * S * 2 <= sms && nk_all / (S * 2) >= 4)
        S *= 2;
    const int kslice = (nk_all + S - 1) / S * kBK;

    GemmParams p;
    p.scales = scales;
    p.zp = zp;
    p.Y = reinterpret_cast<__half *>(Y);
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    (void)scale_f16;   // the entry point admits fp16 scales only
    p.BN = BN;
    p.tmem_cols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
    p.S = S;
    p.kslice = kslice;
    // rings: 4 fp16 weight tiles, 8 packed tiles, as many X tiles as fit (<= 8)
    const int fixed = kWS * kWBytes + kPS * kPBytes;
    int xstages = (224 * 1024 - fixed) / (BN * 128);
    if (xstages > 8) xstages = 8;
    if (xstages < 2) xstages = 2;
    const size_t ring_bytes = (size_t)fixed + (size_t)xstages * BN * 128;
    // the cluster reduction reuses the rings: the parts received from the
    // other S - 1 ranks ([per owned chunk][128][16] fp32 each) and the owned
    // chunks' fp16 tile
    const size_t chunks = (size_t)BN / 16, per = (chunks + S - 1) / S;
    if (S > 1 && ring_bytes < (size_t)(S - 1) * per * kChunkBytes + per * 16 * kBM * 2)
        return fail(MNB_ERR_SHAPE, "mnb_gemm: reduction buffer does not fit");
    p.xstages = xstages;
    const size_t smem = 1024 + ring_bytes + 8 * (2 * kPS + 2 * kWS + 2 * xstages + 2) + 16;
    if (smem > 232448)
        return fail(MNB_ERR_SHAPE, "mnb_gemm: shared memory plan too large");

    CUtensorMap xmap, wmap;
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)BN};
        const cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(X), gdim, gstride, box,
                             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled (X) failed (%d)", (int)cr);
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)(K / 2)};
        const cuuint32_t box[2] = {32, (cuuint32_t)kBM};
        const cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), gdim, gstride,
                             box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled (W) failed (%d)", (int)cr);
    }

    // Y [M][N] fp16: the epilogue's TMA stores, box [BN tokens][128 rows]
    // (whole tiles) or [16 tokens][128 rows] (chunks of a split tile)
    CUtensorMap ymap;
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)N, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)N * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kBM, (cuuint32_t)(S > 1 ? 16 : BN)};
        const cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&ymap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Y, gdim, gstride, box, estride,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemm: cuTensorMapEncodeTiled (Y) failed (%d)", (int)cr);
    }

    static int configured[kMaxDevices] = {};
    {
        cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(gemm_kernel), (int)smem, configured);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemm: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_tiles * S), (unsigned)mt, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (S > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)S;
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel, xmap, wmap, ymap, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemm: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

int tune_gemm(int min_bn, int max_bn, int max_split) {
    if (min_bn < 16 || max_bn > 256 || min_bn > max_bn || max_split < 1 || max_split > kMaxCluster)
        return MNB_ERR_INVALID_ARG;
    g_gemm_min_bn = min_bn;
    g_gemm_max_bn = max_bn;
    g_gemm_max_split = max_split;
    return MNB_OK;
}

int read_device_status(unsigned *out, int clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_mnb_status, sizeof(unsigned));
    if (e == cudaSuccess) {
        int rc = read_gemv_status(out, clear);
        if (!rc)
            rc = read_res_status(out, clear);
        if (!rc)
            rc = read_chain_status(out, clear);
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

// Tuning hooks: smallest (and largest) token tile the tile heuristic may choose
// (16..256) and the largest cluster split along K (1..8).  Not part of the
// stable ABI.
extern "C" MNB_API int mnb_tune_gemm(int min_bn, int max_split) {
    return mnb::tune_gemm(min_bn, min_bn > mnb::g_gemm_max_bn ? min_bn : mnb::g_gemm_max_bn, max_split);
}
extern "C" MNB_API int mnb_tune_gemm_tiles(int min_bn, int max_bn, int max_split) {
    return mnb::tune_gemm(min_bn, max_bn, max_split);
}
