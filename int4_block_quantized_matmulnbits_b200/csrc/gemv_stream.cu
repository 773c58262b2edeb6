// gemv_stream.cu -- decode-shaped MatMulNBits with fp16 activations, 1 <= M <= 8:
// Y[M][N] = X[M][K] . dequant(W)^T, the per-token decoder step of
// "Qwen3-ASR-0.6B -- ONNX for the browser" ("Graph contracts": decoder_step) and
// of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)" (decoder_step_int4).
//
// Every weight byte is read once, so the kernel is shaped around two facts of a
// decode step on B200: the weights stream from HBM, and a step is a CHAIN of
// dependent launches, each of which should be streaming before its
// predecessor has finished.
//   * One CTA per SM (grid <= SM count) using under half of an SM's shared
//     memory and registers, so that under programmatic dependent launch the
//     NEXT call's CTA sits beside this one and fills its own ring meanwhile.
//   * Work unit: a tile of 16 weight rows x one box of 256 k.  A CTA takes
//     groups of TPC tiles; W = 8 / TPC warps share a tile, warp wk taking
//     boxes wk, wk + W, wk + 2W, ...  So one ring stage (TPC tiles x W
//     consecutive boxes) is three dense rectangles of the stored tensors.
//   * Warp 8 is the producer.  It never waits for the previous kernel (the
//     weights do not depend on it): per stage one TMA each for the packed
//     bytes (128-byte swizzle), the scales and the zero points, completing
//     on the stage's mbarrier, kStages stages deep.
//   * Warps 0-7 consume.  They wait for the previous kernel (griddepcontrol),
//     take their activation fragments straight from global memory, then per
//     stage each lane unpacks 2 rows x 64 k of its warp's box to the exact
//     fp16 values q - zp ((nibble | 0x6400) - (1024 + zp) for low nibbles,
//     (16 q + 1024)/16 - (64 + zp) by one fused multiply-add for high
//     nibbles), rounds them once times the fp16 scale -- the value
//     fp16_rn((q - zp) * scale) the dequantizer writes -- and multiplies with
//     X on the tensor cores (mma.sync m16n8k16, fp32 accumulation): 13
//     integer/half instructions per 8 weights.  (Scaling after the MMA would
//     not work: an MMA sums over the four lanes of a quad, which hold four
//     different blocks.)
//   * The W partial sums of a tile meet without a CTA barrier: each warp
//     parks its partial in a shared slot and bumps the tile's counter; the
//     last of the W warps adds the partials in fixed order and stores Y, so
//     results do not depend on timing.
// Requirements (else the caller uses the general kernel): M <= 8, K % 256 ==
// 0, and the scale / zero-point rows must be TMA-addressable (their row pitch
// a multiple of 16 bytes, one stage's slice at least 16 bytes wide).
// Every mbarrier wait is bounded in time; past the limit the kernel records the
// failure in the decode status word, stops issuing, drains what it issued and
// exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace mnb {

namespace {

constexpr int kCons = 8;                       // consumer warps
constexpr int kThreads = (kCons + 1) * 32;     // + producer warp
constexpr int kRows = 16;
constexpr int kBoxK = 256;
constexpr int kBoxBytes = kRows * 128;         // packed bytes of one box
constexpr int kMaxStages = 6;
constexpr int kPkBytes = kCons * kBoxBytes;    // 16 KB of packed weights per stage
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

struct StreamParams {
    const __half *X;
    __half *Y;
    int M, N, K;
    int T, B;            // row tiles, boxes per row (K / 256)
    int W, TPC, nbx;     // warps per tile, tiles per group, stages per group
    int ngroups;
    int sc_pitch;        // bytes of one row of a stage's scale rectangle (W boxes)
    int zp_pitch;        // bytes of one row of a stage's zero-point rectangle
    int sc_off, zp_off;  // offsets of the scale / zero-point rectangles in a stage
    int stage_bytes;
    int tx_bytes;        // bytes the three copies of one stage deliver
    int nstages, nred;   // ring depth, partial-sum slots
    int MP;              // partial-sum columns kept per row (M rounded up to even)
};

}  // namespace

__device__ unsigned g_stream_status = 0;

namespace {

__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, bool &dead, volatile int *abort_flag) {
    if (dead)
        return false;
    unsigned long long t0 = 0;
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 1023) == 0) {   // a long wait: look at the clock and the abort flag
            if (*abort_flag) {
                dead = true;
                return false;
            }
            const unsigned long long now = globaltimer();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitLimitNs) {
                dead = true;
                *abort_flag = 1;
                atomicOr(&g_stream_status, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *map, uint32_t bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}


// One 32-bit word of nibbles e0..e7 of a row -> the fp16 pairs (e0,e4) (e1,e5)
// (e2,e6) (e3,e7) of fp16_rn((q - zp) * scale).  q - zp is exact first:
// (nibble | 0x6400) = 1024 + q minus Z = 1024 + zp for low nibbles, and
// (16 q + 1024) / 16 - (64 + zp) by one fused multiply-add (Zn = -(64 + zp))
// for high nibbles; one multiply by the fp16 scale s2 then rounds once.
__device__ __forceinline__ void dq_word(uint32_t w, uint32_t Z, uint32_t Zn, uint32_t s2, uint32_t &a0,
                                        uint32_t &a1, uint32_t &a2, uint32_t &a3) {
    const half2 sixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    const half2 s = u32_as_h2(s2);
    const uint32_t w8 = w >> 8;
    a0 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s));
    a1 = h2_as_u32(__hmul2(__hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth, u32_as_h2(Zn)), s));
    a2 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w8, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s));
    a3 = h2_as_u32(__hmul2(__hfma2(u32_as_h2(lop3_and_or(w8, 0x00F000F0u, 0x64006400u)), sixteenth, u32_as_h2(Zn)), s));
}

// X fragments of one box for token g: for chunk h (0, 1) and word w (0..3) of the
// lane's chunk 2c + h, the pairs (x0,x4) (x1,x5) | (x2,x6) (x3,x7) of the 8
// activations k0 .. k0+7, k0 = box*256 + (2c+h)*32 + 8w.
struct XFrag {
    uint32_t v[2][4][4];
};

__device__ __forceinline__ void load_xfrag(XFrag &f, const __half *xrow, bool valid, int box, int c) {
#pragma unroll
    for (int h = 0; h < 2; h++)
#pragma unroll
        for (int w = 0; w < 4; w++) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (valid)
                v = ldg_v4(xrow + box * kBoxK + (2 * c + h) * 32 + 8 * w);
            f.v[h][w][0] = __byte_perm(v.x, v.z, 0x5410);
            f.v[h][w][1] = __byte_perm(v.x, v.z, 0x7632);
            f.v[h][w][2] = __byte_perm(v.y, v.w, 0x5410);
            f.v[h][w][3] = __byte_perm(v.y, v.w, 0x7632);
        }
}

}  // namespace

namespace {

template <bool BS64, bool ZP, bool SF32>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap pmap, const __grid_constant__ CUtensorMap smap,
                       const __grid_constant__ CUtensorMap zmap, const StreamParams p) {
    constexpr int kBpb = BS64 ? 4 : 8;                   // blocks per box
    constexpr int kSel = SF32 ? 4 : 2;                   // scale element bytes
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int G = gridDim.x;
    const int R = p.nstages;
    const int my_groups = (p.ngroups > (int)blockIdx.x) ? (p.ngroups - (int)blockIdx.x + G - 1) / G : 0;
    const int total = my_groups * p.nbx;   // stages of this CTA

    // layout (1024-aligned): R stages | nred x [8 warps][16 rows][MP cols] f32 |
    // X [8 warps][nbx*M*512] | counters [nred][8] | barriers | abort flag
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *bp = smem_raw + (base - smem_u32(smem_raw));
    float *red = reinterpret_cast<float *>(bp + (size_t)R * p.stage_bytes);
    const int MP = p.MP;   // partial-sum columns kept: M rounded up to even
    unsigned char *xs = reinterpret_cast<unsigned char *>(red + (size_t)p.nred * kCons * kRows * MP);
    const int xs_warp = (p.nbx > 1) ? p.nbx * p.M * 512 : 0;
    int *cnt = reinterpret_cast<int *>(xs + kCons * xs_warp);
    const uint32_t bars = smem_u32(cnt + p.nred * kCons);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bp + (bars - base) + 16 * R);

    if (tid == 0) {
        for (int i = 0; i < R; i++) {
            mbar_init(bars + 8u * i, 1);
            mbar_init(bars + 8u * (R + i), kCons);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < p.nred * kCons; i += kThreads)
        cnt[i] = 0;
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kCons) {
        // ================= producer: weights, scales, zero points (no wait for
        // the previous kernel: none of this is written by it)
        bool dead = false;
        int issued = 0;
        if (lane == 0) {
            int slot = 0, pp = 0, row0 = (int)blockIdx.x * p.TPC * kRows;
            uint32_t phase = 0;
            const int row_step = G * p.TPC * kRows;
            for (int s = 0; s < total; s++) {
                if (s >= R && !bounded_wait(bars + 8u * (uint32_t)(R + slot), phase ^ 1u, dead, abort_flag))
                    break;
                const uint32_t st = base + (uint32_t)(slot * p.stage_bytes);
                const uint32_t fb = bars + 8u * (uint32_t)slot;
                mbar_expect_tx(fb, (uint32_t)p.tx_bytes);
                tma_load_3d(st, &pmap, fb, 0, row0, pp * p.W);
                tma_load_2d(st + (uint32_t)p.sc_off, &smap, fb, pp * p.W * kBpb, row0);
                if (ZP)
                    tma_load_2d(st + (uint32_t)p.zp_off, &zmap, fb, pp * p.W * (kBpb / 2), row0);
                issued = s + 1;
                if (++slot == R) { slot = 0; phase ^= 1u; }
                if (++pp == p.nbx) { pp = 0; row0 += row_step; }
            }
        }
        __syncwarp();
        __syncthreads();
        if (lane == 0 && *abort_flag) {
            // let every copy still in flight land before shared memory goes away
            for (int s = (issued > R ? issued - R : 0); s < issued; s++) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(bars + 8u * (uint32_t)(s % R), (uint32_t)((s / R) & 1)) &&
                       globaltimer() - t0 < kWaitLimitNs) {
                }
            }
        }
        return;
    }

    // ================= consumers
    bool dead = false;
    pdl_wait();   // X is the previous kernel's output
    const int wt = warp / p.W, wk = warp - wt * p.W;   // tile slot in the group, K interleave
    const bool tok = g < p.M;
    const __half *xrow = p.X + (size_t)(tok ? g : 0) * p.K;
    unsigned char *xw = xs + warp * xs_warp;
    XFrag f;
    if (p.nbx == 1) {
        load_xfrag(f, xrow, tok && wk < p.B, wk < p.B ? wk : 0, c);
    } else {
        // this warp's boxes wk, wk + W, ... are the same in every group: keep
        // their fragments (real tokens only) in the warp's own shared memory
        for (int pp = 0; pp < p.nbx; pp++) {
            const int j = pp * p.W + wk;
            load_xfrag(f, xrow, tok && j < p.B, j < p.B ? j : 0, c);
            if (tok)
#pragma unroll
                for (int h = 0; h < 2; h++)
#pragma unroll
                    for (int w = 0; w < 4; w++)
                        *reinterpret_cast<uint4 *>(xw + (((pp * 8 + h * 4 + w) * p.M + g) * 4 + c) * 16) =
                            make_uint4(f.v[h][w][0], f.v[h][w][1], f.v[h][w][2], f.v[h][w][3]);
        }
        __syncwarp();
    }

    const int box_off = (wk * p.TPC + wt) * kBoxBytes;
    const int row_g = wt * kRows + g;                  // this lane's first row in the stage rectangles
    // byte offsets inside a stage: packed chunks 2c, 2c+1 of rows g and g+8
    // (128-byte swizzle), the lane's scales and zero points
    const int pk_off0 = box_off + g * 128 + (((2 * c) ^ g) << 4);
    const int pk_off1 = box_off + g * 128 + (((2 * c + 1) ^ g) << 4);
    const int sc_lane = p.sc_off + row_g * p.sc_pitch + wk * (kBpb * kSel) + (BS64 ? c : 2 * c) * kSel;
    const int zp_lane = p.zp_off + row_g * p.zp_pitch + wk * (kBpb / 2) + (BS64 ? (c >> 1) : c);
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    int slot = 0, pp = 0, rslot = 0, tile = (int)blockIdx.x * p.TPC + wt;
    uint32_t phase = 0;
    for (int s = 0; s < total; s++) {
        const int j = pp * p.W + wk;
        if (p.nbx > 1) {
#pragma unroll
            for (int h = 0; h < 2; h++)
#pragma unroll
                for (int w = 0; w < 4; w++) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (tok)
                        v = *reinterpret_cast<const uint4 *>(xw + (((pp * 8 + h * 4 + w) * p.M + g) * 4 + c) * 16);
                    f.v[h][w][0] = v.x; f.v[h][w][1] = v.y; f.v[h][w][2] = v.z; f.v[h][w][3] = v.w;
                }
        }
        const bool ok = bounded_wait(bars + 8u * (uint32_t)slot, phase, dead, abort_flag);
        if (ok && tile < p.T && j < p.B) {
            const unsigned char *st = bp + (size_t)slot * p.stage_bytes;
            const unsigned char *sc0 = st + sc_lane;
            const unsigned char *sc8 = sc0 + 8 * p.sc_pitch;
            // fp16 scales of rows g and g+8 for chunks 2c, 2c+1, each in both halves
            uint32_t sg[2], sg8[2];
            if (!BS64) {
                if (SF32) {
                    const float2 a = *reinterpret_cast<const float2 *>(sc0);
                    const float2 b = *reinterpret_cast<const float2 *>(sc8);
                    sg[0] = h2_as_u32(__float2half2_rn(a.x)); sg[1] = h2_as_u32(__float2half2_rn(a.y));
                    sg8[0] = h2_as_u32(__float2half2_rn(b.x)); sg8[1] = h2_as_u32(__float2half2_rn(b.y));
                } else {
                    const uint32_t a = *reinterpret_cast<const uint32_t *>(sc0);
                    const uint32_t b = *reinterpret_cast<const uint32_t *>(sc8);
                    sg[0] = __byte_perm(a, a, 0x1010); sg[1] = __byte_perm(a, a, 0x3232);
                    sg8[0] = __byte_perm(b, b, 0x1010); sg8[1] = __byte_perm(b, b, 0x3232);
                }
            } else {
                if (SF32) {
                    sg[0] = sg[1] = h2_as_u32(__float2half2_rn(*reinterpret_cast<const float *>(sc0)));
                    sg8[0] = sg8[1] = h2_as_u32(__float2half2_rn(*reinterpret_cast<const float *>(sc8)));
                } else {
                    const uint32_t a = *reinterpret_cast<const unsigned short *>(sc0);
                    const uint32_t b = *reinterpret_cast<const unsigned short *>(sc8);
                    sg[0] = sg[1] = a | (a << 16);
                    sg8[0] = sg8[1] = b | (b << 16);
                }
            }
            // zero points of rows g and g+8 for chunks 2c, 2c+1
            uint32_t zg[2] = {8u, 8u}, zg8[2] = {8u, 8u};
            if (ZP) {
                const unsigned char *z0 = st + zp_lane;
                const unsigned char *z8 = z0 + 8 * p.zp_pitch;
                if (!BS64) {
                    const uint32_t a = z0[0], b = z8[0];
                    zg[0] = a & 15u; zg[1] = a >> 4; zg8[0] = b & 15u; zg8[1] = b >> 4;
                } else {
                    const int sh = (c & 1) * 4;
                    zg[0] = zg[1] = (uint32_t)(z0[0] >> sh) & 15u;
                    zg8[0] = zg8[1] = (uint32_t)(z8[0] >> sh) & 15u;
                }
            }
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const unsigned char *pa = st + (h ? pk_off1 : pk_off0);
                const uint4 va = *reinterpret_cast<const uint4 *>(pa);
                const uint4 vb = *reinterpret_cast<const uint4 *>(pa + 8 * 128);
                // the zero point lands in bits that the constants leave clear: one IMAD each
                const uint32_t Za = zg[h] * 0x00010001u + 0x64006400u, Zb = zg8[h] * 0x00010001u + 0x64006400u;
                const uint32_t Zna = zg[h] * 0x00100010u + 0xD400D400u, Znb = zg8[h] * 0x00100010u + 0xD400D400u;
                const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
                const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                for (int w = 0; w < 4; w++) {
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    dq_word(wa[w], Za, Zna, sg[h], a0, a1, a2, a3);
                    dq_word(wb[w], Zb, Znb, sg8[h], b0, b1, b2, b3);
                    float *acc = h ? acc1 : acc0;
                    mma16816(acc, a0, b0, a1, b1, f.v[h][w][0], f.v[h][w][1]);
                    mma16816(acc, a2, b2, a3, b3, f.v[h][w][2], f.v[h][w][3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars + 8u * (uint32_t)(R + slot));
        if (++slot == R) { slot = 0; phase ^= 1u; }

        if (++pp == p.nbx) {
            pp = 0;
            // ---- end of a group: park this warp's partial sums; the last of the
            // tile's W warps adds them in fixed order and stores Y
            float *rb = red + (size_t)(rslot * kCons + warp) * (kRows * MP);
            if (2 * c < MP) {
                rb[g * MP + 2 * c] = acc0[0] + acc1[0];
                rb[g * MP + 2 * c + 1] = acc0[1] + acc1[1];
                rb[(g + 8) * MP + 2 * c] = acc0[2] + acc1[2];
                rb[(g + 8) * MP + 2 * c + 1] = acc0[3] + acc1[3];
            }
#pragma unroll
            for (int e = 0; e < 4; e++) acc0[e] = acc1[e] = 0.f;
            __threadfence_block();
            __syncwarp();
            int old = 0;
            if (lane == 0)
                old = atomicAdd(&cnt[rslot * kCons + wt], 1);
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == p.W - 1 && 2 * c < MP) {
                __threadfence_block();
                const float *src = red + (size_t)(rslot * kCons + wt * p.W) * (kRows * MP);
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                for (int w = 0; w < p.W; w++) {
                    const float *sw = src + w * (kRows * MP);
                    v[0] += sw[g * MP + 2 * c];
                    v[1] += sw[g * MP + 2 * c + 1];
                    v[2] += sw[(g + 8) * MP + 2 * c];
                    v[3] += sw[(g + 8) * MP + 2 * c + 1];
                }
                const int n0 = tile * kRows + g;
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int m = 2 * c + (e & 1), n = n0 + 8 * (e >> 1);
                    if (m < p.M && n < p.N && tile < p.T)
                        p.Y[(size_t)m * p.N + n] = __float2half_rn(v[e]);
                }
            }
            if (old == p.W - 1 && lane == 0)
                cnt[rslot * kCons + wt] = 0;   // after lane 0's own reads; the other lanes
                                               // finish theirs before this warp's next group
            if (++rslot == p.nred) rslot = 0;
            tile += G * p.TPC;
        }
    }
    __syncthreads();   // pairs with the producer's: it drains after a timeout
}

constexpr size_t kSmemCap = 110 * 1024;   // under half an SM: the next call's CTA fits beside this one

template <bool BS64, bool ZP, bool SF32>
int launch_stream(const CUtensorMap maps[3], const StreamParams &p, int grid, size_t smem, unsigned flags,
                  cudaStream_t s) {
    auto fn = gemv_stream_kernel<BS64, ZP, SF32>;
    static int configured[kMaxDevices] = {};
    {
        cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(fn), (int)smem, configured);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (flags & MNB_FLAG_PDL) ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, maps[0], maps[1], maps[2], p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

}  // namespace

// Returns 1 (and launches nothing) when the shape or alignment is outside what
// this kernel serves; the caller then uses the general decode kernel.
int launch_gemv_stream(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                       void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s) {
    const bool bs64 = (bs == 64), has_zp = (zp != nullptr), sf32 = !scale_f16;
    if (M < 1 || M > 8 || K % kBoxK != 0)
        return 1;
    const int nb = K / bs, zpb = (nb + 1) / 2;
    const int sel = sf32 ? 4 : 2, bpb = bs64 ? 4 : 8, zbb = bpb / 2;
    // TMA-addressable scale / zero-point rows
    if (!aligned(scales, 16) || ((size_t)nb * sel) % 16 != 0)
        return 1;
    if (has_zp && (!aligned(zp, 16) || zpb % 16 != 0))
        return 1;
    EncodeTiledFn encode = tensor_map_encoder();
    if (!encode)
        return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled unavailable");
    const int sms = device_sm_count();

    StreamParams p;
    p.X = reinterpret_cast<const __half *>(X);
    p.Y = reinterpret_cast<__half *>(Y);
    p.M = M; p.N = N; p.K = K;
    p.T = (N + kRows - 1) / kRows;
    p.B = K / kBoxK;

    // W warps per tile: fewest stages on the busiest CTA; ties go to the larger W
    int best = -1, best_cost = 0;
    for (int W = 8; W >= 1; W >>= 1) {
        if (W > p.B || (W * bpb * sel) % 16 != 0 || (has_zp && (W * zbb) % 16 != 0))
            continue;
        const int TPC = kCons / W, nbx = (p.B + W - 1) / W;
        const int ngroups = (p.T + TPC - 1) / TPC;
        const int G = ngroups < sms ? ngroups : sms;
        const int cost = ((ngroups + G - 1) / G) * nbx;
        if (nbx > 1 && (size_t)kCons * nbx * M * 512 > 24 * 1024)
            continue;
        if (best < 0 || cost < best_cost) {
            best = W;
            best_cost = cost;
        }
    }
    if (best < 0)
        return 1;
    p.W = best;
    p.TPC = kCons / p.W;
    p.nbx = (p.B + p.W - 1) / p.W;
    p.ngroups = (p.T + p.TPC - 1) / p.TPC;
    const int rows = p.TPC * kRows;
    p.sc_pitch = p.W * bpb * sel;
    p.zp_pitch = has_zp ? p.W * zbb : 0;
    p.sc_off = kPkBytes;
    p.zp_off = kPkBytes + rows * p.sc_pitch;
    p.stage_bytes = (p.zp_off + rows * p.zp_pitch + 1023) & ~1023;
    p.tx_bytes = kPkBytes + rows * p.sc_pitch + rows * p.zp_pitch;
    p.MP = (M + 1) & ~1;
    const int grid = p.ngroups < sms ? p.ngroups : sms;
    const size_t xs = (p.nbx > 1) ? (size_t)kCons * p.nbx * M * 512 : 0;
    int R = kMaxStages;
    size_t smem = 0;
    for (; R >= 2; R--) {
        p.nstages = R;
        p.nred = R + 1;
        smem = 1024 + (size_t)R * p.stage_bytes + (size_t)p.nred * kCons * kRows * p.MP * 4 + xs +
               (size_t)p.nred * kCons * 4 + (size_t)2 * R * 8 + 16;
        if (smem <= kSmemCap)
            break;
    }
    if (R < 2)
        return 1;

    CUtensorMap maps[3];
    {   // packed bytes viewed as [box j][row n][128 bytes]: one stage = TPC*16 rows x W boxes
        const cuuint64_t gdim[3] = {128, (cuuint64_t)N, (cuuint64_t)p.B};
        const cuuint64_t gstride[2] = {(cuuint64_t)(K / 2), 128};
        const cuuint32_t box[3] = {128, (cuuint32_t)rows, (cuuint32_t)p.W};
        const cuuint32_t estride[3] = {1, 1, 1};
        if (encode(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(packed), gdim, gstride, box,
                   estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled (weights) failed");
    }
    {   // scales [N][nb]
        const cuuint64_t gdim[2] = {(cuuint64_t)nb, (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)nb * sel};
        const cuuint32_t box[2] = {(cuuint32_t)(p.W * bpb), (cuuint32_t)rows};
        const cuuint32_t estride[2] = {1, 1};
        if (encode(&maps[1], sf32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                   const_cast<void *>(scales), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled (scales) failed");
    }
    if (has_zp) {   // zero points [N][zpb] bytes
        const cuuint64_t gdim[2] = {(cuuint64_t)zpb, (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)zpb};
        const cuuint32_t box[2] = {(cuuint32_t)(p.W * zbb), (cuuint32_t)rows};
        const cuuint32_t estride[2] = {1, 1};
        if (encode(&maps[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(zp), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled (zero points) failed");
    } else {
        maps[2] = maps[1];   // unused
    }
#define MNB_ST(B_, Z_, S_) return launch_stream<B_, Z_, S_>(maps, p, grid, smem, flags, s)
    if (bs64) {
        if (has_zp) { if (sf32) MNB_ST(true, true, true); else MNB_ST(true, true, false); }
        else { if (sf32) MNB_ST(true, false, true); else MNB_ST(true, false, false); }
    } else {
        if (has_zp) { if (sf32) MNB_ST(false, true, true); else MNB_ST(false, true, false); }
        else { if (sf32) MNB_ST(false, false, true); else MNB_ST(false, false, false); }
    }
#undef MNB_ST
}

int read_stream_status(unsigned *out, int clear) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_stream_status, sizeof(unsigned));
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_stream_status, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_device_status: %s", cudaGetErrorString(e));
    *out |= v;
    return MNB_OK;
}

}  // namespace mnb
