// gemv_tc.cu -- decode-shaped MatMulNBits with fp16 activations (1 <= M <= 32):
// Y[M][N] = X[M][K] . dequant(W)^T, the per-token decoder step of
// "Qwen3-ASR-0.6B -- ONNX for the browser" ("Graph contracts": decoder_step)
// and of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)" (decoder_step_int4).
//
// HBM-bound: every weight byte is read once, so the kernel is built to keep the
// memory system full while the SM does the int4 -> fp16 work.
//   * Weights move by TMA.  A 2D tensor map views the packed bytes as
//     [N rows][K/2 bytes]; one box is 16 rows x 128 bytes (256 k), landing in
//     shared memory with the 128-byte swizzle.  Each warp owns a ring of
//     kDepth boxes with one mbarrier each; lane 0 keeps kDepth boxes in
//     flight, so a whole SM holds tens of KB of outstanding weight traffic
//     with a handful of instructions and no registers.
//   * The first boxes are requested BEFORE griddepcontrol.wait: under
//     programmatic dependent launch the weight stream of this kernel starts
//     while the previous kernel is still finishing.  X is read after the wait.
//   * Thread (g = lane/4, c = lane%4) owns rows g and g+8 of the warp's 16-row
//     tile and, in every box, the 16-byte chunks 2c and 2c+1 of both rows; the
//     swizzle makes these shared-memory reads conflict-free.
//   * Unpack + dequant in registers: (nibble | 0x6400) is the fp16 1024+q
//     exactly; subtracting 1024+zp leaves q-zp exactly; one multiply gives
//     fp16_rn((q - zp) * scale), the same value the dequantizer writes.  High
//     nibbles come out as 1024+16q and stay at 16x scale (exact); the
//     activations they meet are staged as x/16 (exact).  So 8 weights cost one
//     shift, four LOP3, four HSUB2 and four HMUL2.
//   * The hot loop is compiled per configuration (block size, zero points,
//     scale type) and carries no runtime branches.
//   * mma.sync m16n8k16 (fp32 accumulation) takes the 16 rows as M and the
//     tokens as N, so the multiply-adds leave the CUDA cores to the unpack.
//   * Persistent CTAs of 8 warps, two per SM.  When tiles alone cannot occupy
//     the SMs, K is split over W warps of a CTA (shared-memory reduction) and
//     over a cluster of S CTAs (distributed shared memory): no global scratch.
// Every mbarrier wait is bounded in time; past the limit the kernel records the
// failure in a device status word, drains its copies and exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "mnb_tune.h"

namespace mnb {

namespace {

__device__ unsigned g_gemv_status = 0;

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;
constexpr int kBoxK = 256;                 // k per TMA box
constexpr int kBoxBytes = kRows * 128;     // 16 rows x 128 packed bytes
constexpr int kDepth = 4;                  // boxes in flight per warp
constexpr int kMaxCluster = 8;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr size_t kArgmaxWsHeader = 256;    // the CTA counter, then the per-CTA partials

struct ArgmaxArgs {
    int32_t *ids;
    float *max_out;
    void *workspace;
};

struct TcParams {
    const void *X;
    const void *scales;
    const uint8_t *zp;
    __half *Y;
    int M, N, K;
    int bs_shift, nb, zpb, scale_f16, scale_pair;
    int S;            // CTAs per cluster (K split across CTAs)
    int W;            // warps per tile inside a CTA (K split across warps)
    int nbx_w;        // boxes in one warp's K slice
    int kcta;         // k covered by one CTA = W * nbx_w * kBoxK
    int rounds;       // tile rounds per CTA (split mode)
    int nclusters;    // gridDim.x / S
    int xs_stride;    // bytes per token row of staged X
    int ntiles;       // ceil(N / 16)
    int independent;  // W == 1 && S == 1: each warp walks tiles on its own
    // SwiGLU epilogue: weight rows come in 16-row groups of 8 gate rows and the
    // 8 up rows of the same outputs; Y[m][8t + i] = silu(gate) * up, N / 2 columns
    int swiglu;
    // greedy decoding (independent mode only): ids[m] = first n of max Y[m][n]
    int argmax;
    int *ids;             // [M]
    float *max_out;       // [M] or null
    uint2 *ws_part;       // [gridDim.x][M] (value bits, index) per CTA
    unsigned *ws_count;   // CTAs done; the last one resets it to 0
};



__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}


// Bounded wait on a warp-private mbarrier.  After the first timeout (*dead set)
// it returns at once, so the warp runs to the end without waiting again.
__device__ __forceinline__ void box_wait(uint32_t bar, uint32_t parity, bool &dead) {
    if (dead || mbar_try_wait(bar, parity))
        return;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(bar, parity))
            return;
        if ((i & 255) == 0 && globaltimer() - t0 > kWaitLimitNs) {
            dead = true;
            atomicOr(&g_gemv_status, 1u);
            return;
        }
    }
}

// Scale (fp16 bits) and zero point of the two chunks (2c, 2c+1) a thread
// dequantizes in one box, for one row.
struct ChunkParams {
    uint32_t s[2];
    uint32_t z[2];
};

// Where a thread's scales and zero points of the current tile live; moving to
// the next box is a pointer increment.
struct ParamCursor {
    const uint8_t *s;     // scale of the thread's first block in this box (row g)
    const uint8_t *z;     // its zero-point byte (row g)
    int k0;               // k of the thread's first chunk in this box
    bool ok0, ok1;        // rows g, g+8 inside N
};

template <class C>
__device__ __forceinline__ void param_tile(const TcParams &p, ParamCursor &q, int tile, int g, int kfirst) {
    const int n = tile * kRows + g;
    const int b0 = kfirst >> (C::bs64 ? 6 : 5);
    q.k0 = kfirst;
    q.ok0 = n < p.N;
    q.ok1 = n + 8 < p.N;
    q.s = reinterpret_cast<const uint8_t *>(p.scales) + ((int64_t)n * p.nb + b0) * ((C::smode == 0) ? 2 : (p.scale_f16 ? 2 : 4));
    q.z = C::zp ? p.zp + (int64_t)n * p.zpb + (b0 >> 1) : nullptr;
}

// Configuration of the hot loop, fixed at compile time so that it carries no
// runtime branches: block size 64?  zero points present?  SMODE 0 = fp16 scales
// read as aligned pairs (block 32) or singly (block 64); SMODE 1 = anything else
// (fp32 scales, or fp16 scales an aligned pair load cannot serve).
template <bool BS64, bool ZP, int SMODE>
struct Cfg {
    static constexpr bool bs64 = BS64, zp = ZP;
    static constexpr int smode = SMODE;
};

__device__ __forceinline__ uint32_t h16_at(const TcParams &p, const uint8_t *ptr) {
    if (p.scale_f16)
        return __ldg(reinterpret_cast<const unsigned short *>(ptr));
    return __half_as_ushort(__float2half_rn(__ldg(reinterpret_cast<const float *>(ptr))));
}

// Parameters of the box at the cursor for row g (r = 0) or g+8 (r = 1).
template <class C>
__device__ __forceinline__ ChunkParams params_at(const TcParams &p, const ParamCursor &q, int r) {
    ChunkParams c;
    c.s[0] = c.s[1] = 0;
    c.z[0] = c.z[1] = 8;
    if (!(r ? q.ok1 : q.ok0) || q.k0 >= p.K)
        return c;
    const int ssz = (C::smode == 0) ? 2 : (p.scale_f16 ? 2 : 4);
    const uint8_t *sp = q.s + (r ? (int64_t)8 * p.nb * ssz : 0);
    if (!C::bs64) {   // block 32: chunks 2c, 2c+1 are blocks b0, b0+1 (b0 even)
        if (C::smode == 0) {
            const uint32_t pair = __ldg(reinterpret_cast<const unsigned int *>(sp));
            c.s[0] = pair & 0xFFFFu;
            c.s[1] = pair >> 16;
        } else {
            c.s[0] = h16_at(p, sp);
            c.s[1] = (q.k0 + 32 < p.K) ? h16_at(p, sp + ssz) : 0u;
        }
        if (C::zp) {
            const uint32_t zb = __ldg(q.z + (r ? (int64_t)8 * p.zpb : 0));
            c.z[0] = zb & 15u;
            c.z[1] = zb >> 4;
        }
    } else {          // block 64: both chunks in one block
        c.s[0] = c.s[1] = (C::smode == 0) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(sp))
                                          : h16_at(p, sp);
        if (C::zp) {
            const uint32_t zb = __ldg(q.z + (r ? (int64_t)8 * p.zpb : 0));
            c.z[0] = c.z[1] = ((q.k0 >> 6) & 1) ? (zb >> 4) : (zb & 15u);
        }
    }
    return c;
}

template <class C>
__device__ __forceinline__ void param_next_box(const TcParams &p, ParamCursor &q) {
    // one box = 256 k = 8 blocks of 32 or 4 of 64
    constexpr int nblk = C::bs64 ? 4 : 8;
    q.s += nblk * ((C::smode == 0) ? 2 : (p.scale_f16 ? 2 : 4));
    if (C::zp) q.z += nblk >> 1;
    q.k0 += kBoxK;
}


// silu(x) = x * sigmoid(x), in fp32.
__device__ __forceinline__ float silu(float x) { return x / (1.0f + __expf(-x)); }

// (value, index) pairs ordered by value, then by the SMALLER index: the greedy
// token is the first maximum.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void warp_best(float &v, int &i, unsigned mask_lanes) {
    for (unsigned o = 16; o >= 1; o >>= 1) {
        if (!(mask_lanes & o))
            continue;
        const float ov = __shfl_xor_sync(0xffffffffu, v, (int)o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, (int)o);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

// Greedy decoding epilogue: the warp's best per token (lanes with one c hold
// one token pair), then the CTA's, parked in the workspace; the last CTA to
// finish reduces all CTAs' partials and resets the counter.
template <int NT>
__device__ void argmax_finish(const TcParams &p, float (&best_v)[NT][2], int (&best_i)[NT][2], uint2 *sb, int warp,
                              int lane, int g, int c, int tid) {
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int jj = 0; jj < 2; jj++) {
            float v = best_v[t][jj];
            int i = best_i[t][jj];
            warp_best(v, i, 4u | 8u | 16u);   // over g: the 8 lanes that share c
            const int m = 8 * t + 2 * c + jj;
            if (g == 0 && m < p.M)
                sb[warp * 16 + m] = make_uint2(__float_as_uint(v), (unsigned)i);
        }
    __syncthreads();
    __shared__ int s_last;
    if (tid < p.M) {
        float v = -INFINITY;
        int i = 0x7fffffff;
        for (int w = 0; w < kWarps; w++) {
            const uint2 e = sb[w * 16 + tid];
            if (better(__uint_as_float(e.x), (int)e.y, v, i)) {
                v = __uint_as_float(e.x);
                i = (int)e.y;
            }
        }
        p.ws_part[(size_t)blockIdx.x * p.M + tid] = make_uint2(__float_as_uint(v), (unsigned)i);
        __threadfence();
    }
    __syncthreads();
    if (tid == 0)
        s_last = (atomicAdd(p.ws_count, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    for (int m = 0; m < p.M; m++) {
        float v = -INFINITY;
        int i = 0x7fffffff;
        for (int b = tid; b < (int)gridDim.x; b += kThreads) {
            const uint2 e = __ldcg(p.ws_part + (size_t)b * p.M + m);
            if (better(__uint_as_float(e.x), (int)e.y, v, i)) {
                v = __uint_as_float(e.x);
                i = (int)e.y;
            }
        }
        warp_best(v, i, 31u);
        __syncthreads();   // sb is reused per token
        if (lane == 0)
            sb[warp] = make_uint2(__float_as_uint(v), (unsigned)i);
        __syncthreads();
        if (tid == 0) {
            for (int w = 1; w < kWarps; w++) {
                const uint2 e = sb[w];
                if (better(__uint_as_float(e.x), (int)e.y, v, i)) {
                    v = __uint_as_float(e.x);
                    i = (int)e.y;
                }
            }
            p.ids[m] = i;
            if (p.max_out)
                p.max_out[m] = v;
        }
    }
    if (tid == 0)
        *p.ws_count = 0u;   // ready for the next call
}

template <int NT, class C>
__global__ void __launch_bounds__(kThreads, NT >= 4 ? 1 : 2) gemv_tc_kernel(const __grid_constant__ CUtensorMap wmap,
                                                                           const TcParams p) {
    constexpr int MP = 8 * NT;
    constexpr bool kArgmax = NT <= 2;   // greedy decoding serves M <= 16
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int W = p.W, TPC = kWarps / p.W;
    const int slot = warp / W, wk = warp - slot * W;
    const int rank = (p.S > 1) ? (int)cluster_ctarank() : 0;
    const int cluster = blockIdx.x / p.S;
    const int kcta0 = rank * p.kcta;
    const int kw = kcta0 + wk * p.nbx_w * kBoxK;   // first k of this warp's slice
    const int nqb = p.kcta / kBoxK;                // boxes in the CTA's X range

    // shared memory: boxes (1024-aligned) | X | zero row | red | part | barriers
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *bp = smem_raw + (base - smem_u32(smem_raw));
    unsigned char *xs = bp + kWarps * kDepth * kBoxBytes;
    unsigned char *zrow = xs + p.M * p.xs_stride;   // 512 zero bytes: activations of absent tokens
    float *red = reinterpret_cast<float *>(zrow + 512);
    float *part = red + kWarps * kRows * MP;
    const uint32_t bars = smem_u32(part + kWarps * kRows * MP);
    const uint32_t my_boxes = base + (uint32_t)(warp * kDepth * kBoxBytes);
    const unsigned char *my_boxes_ptr = bp + warp * kDepth * kBoxBytes;
    const uint32_t my_bars = bars + (uint32_t)(warp * kDepth * 8);

    int first_tile, tile_stride, units;
    if (p.independent) {
        const int gw = blockIdx.x * kWarps + warp, G = gridDim.x * kWarps;
        first_tile = gw;
        tile_stride = G;
        units = (p.ntiles > gw) ? (p.ntiles - gw + G - 1) / G : 0;
    } else {
        first_tile = cluster * TPC + slot;
        tile_stride = p.nclusters * TPC;
        units = p.rounds;
    }
    const int total = units * p.nbx_w;

    // ---- weights first: they do not depend on the previous kernel
    int is_tile = first_tile, is_j = 0, is_pos = 0;   // TMA issue cursor (lane 0)
    if (lane == 0) {
        for (int d = 0; d < kDepth; d++)
            mbar_init(my_bars + 8 * d, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int d = 0; d < kDepth && is_pos < total; d++) {
            mbar_expect_tx(my_bars + 8 * d, kBoxBytes);
            tma_load_2d(my_boxes + d * kBoxBytes, &wmap, my_bars + 8 * d, (kw + is_j * kBoxK) / 2, is_tile * kRows);
            ++is_pos;
            if (++is_j == p.nbx_w) { is_j = 0; is_tile += tile_stride; }
        }
    }
    __syncwarp();
    // the first box's scales and zero points are weights too: fetch them before
    // waiting for the previous kernel, so their latency overlaps the wait
    ParamCursor pc;
    param_tile<C>(p, pc, first_tile, g, kw + c * 64);
    ChunkParams pa = params_at<C>(p, pc, 0), pb = params_at<C>(p, pc, 1);   // one box ahead
    pdl_launch_dependents();
    pdl_wait();

    // ---- stage X[0:M, kcta0 : kcta0 + kcta).  Box qb, unit (h, w, c) holds
    // k = qb*256 + (2c+h)*32 + 8w .. +7 as (x0,x4) (x1,x5)/16 (x2,x6) (x3,x7)/16;
    // one thread per 32-k chunk.
    {
        const __half *X = reinterpret_cast<const __half *>(p.X);
        const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
        const int per_tok = nqb * 8;   // chunks
        for (int u = tid; u < p.M * per_tok; u += kThreads) {
            const int m = u / per_tok;
            const int r = u - m * per_tok;
            const int qb = r >> 3, chunk = r & 7;
            const int h = chunk & 1, cc = chunk >> 1;
            const int k = kcta0 + qb * kBoxK + chunk * 32;
            uint4 vv[4];
#pragma unroll
            for (int w = 0; w < 4; w++)   // all four loads in flight before any use
                vv[w] = (k < p.K) ? ldg_v4(X + (int64_t)m * p.K + k + 8 * w) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const uint4 v = vv[w];
                uint4 o;
                o.x = __byte_perm(v.x, v.z, 0x5410);
                o.y = h2_as_u32(__hmul2(u32_as_h2(__byte_perm(v.x, v.z, 0x7632)), sixteenth));
                o.z = __byte_perm(v.y, v.w, 0x5410);
                o.w = h2_as_u32(__hmul2(u32_as_h2(__byte_perm(v.y, v.w, 0x7632)), sixteenth));
                *reinterpret_cast<uint4 *>(xs + m * p.xs_stride + qb * 512 + h * 256 + w * 64 + cc * 16) = o;
            }
        }
        for (int i = tid; i < 128; i += kThreads)
            reinterpret_cast<uint32_t *>(zrow)[i] = 0u;
    }
    __syncthreads();

    // independent MMA accumulator chains per token group: chunk 2c + h, and with
    // one column group also the word parity (shorter dependency chains;
    // measured 1.4 % faster on the 1.7B step at M = 1, slower at M = 16)
    constexpr int kChains = (NT == 1) ? 4 : 2;
    float acc[NT][kChains][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int e = 0; e < 4 * kChains; e++) acc[t][e >> 2][e & 3] = 0.f;

    bool dead = false;
    int tile = first_tile, j = 0, r = 0;
    float best_v[NT][2];   // greedy decoding: the lane's best logit so far for tokens 8t + 2c + jj
    int best_i[NT][2];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int jj = 0; jj < 2; jj++) {
            best_v[t][jj] = -INFINITY;
            best_i[t][jj] = 0x7fffffff;
        }
    for (int pos = 0; pos < total; pos++) {
        int ntile = tile, nj = j + 1;
        if (nj == p.nbx_w) { nj = 0; ntile += tile_stride; }
        if (nj == 0) param_tile<C>(p, pc, ntile, g, kw + c * 64); else param_next_box<C>(p, pc);
        ChunkParams na = pa, nbq = pb;
        if (pos + 1 < total) {
            na = params_at<C>(p, pc, 0);
            nbq = params_at<C>(p, pc, 1);
        }

        const int d = pos % kDepth;
        box_wait(my_bars + 8 * d, (uint32_t)((pos / kDepth) & 1), dead);
        const unsigned char *box = my_boxes_ptr + d * kBoxBytes;
        const int qb = wk * p.nbx_w + j;      // box index inside the CTA's X range
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int chunk = 2 * c + h;
            const uint4 va = *reinterpret_cast<const uint4 *>(box + g * 128 + ((chunk ^ g) << 4));
            const uint4 vb = *reinterpret_cast<const uint4 *>(box + (g + 8) * 128 + ((chunk ^ g) << 4));
            const uint32_t sa = pa.s[h] | (pa.s[h] << 16), sb = pb.s[h] | (pb.s[h] << 16);
            const uint32_t Za = 0x64006400u | (pa.z[h] * 0x00010001u), Zb = 0x64006400u | (pb.z[h] * 0x00010001u);
            const uint32_t Zha = 0x64006400u | (pa.z[h] * 0x00100010u), Zhb = 0x64006400u | (pb.z[h] * 0x00100010u);
            const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
            const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const int tok = g + 8 * t;
                const unsigned char *xa = (tok < p.M) ? xs + tok * p.xs_stride + qb * 512 + h * 256 + c * 16
                                                      : zrow + h * 256 + c * 16;
#pragma unroll
                for (int w = 0; w < 4; w++) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(xa + w * 64);
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    dq_word(wa[w], sa, Za, Zha, a0, a1, a2, a3);
                    dq_word(wb[w], sb, Zb, Zhb, b0, b1, b2, b3);
                    float *ac = acc[t][kChains == 4 ? 2 * h + (w & 1) : h];
                    mma16816(ac, a0, b0, a1, b1, xv.x, xv.y);
                    mma16816(ac, a2, b2, a3, b3, xv.z, xv.w);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && is_pos < total) {
            // box d is free again: refill it with the box kDepth positions ahead
            fence_proxy_async_smem();
            mbar_expect_tx(my_bars + 8 * d, kBoxBytes);
            tma_load_2d(my_boxes + d * kBoxBytes, &wmap, my_bars + 8 * d, (kw + is_j * kBoxK) / 2, is_tile * kRows);
            ++is_pos;
            if (++is_j == p.nbx_w) { is_j = 0; is_tile += tile_stride; }
        }
        pa = na;
        pb = nbq;
        if (nj != 0) {
            j = nj;
            continue;
        }

        // ---- end of a tile (for every warp of the CTA at once in split mode)
        float out[NT][4];
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                out[t][e] = acc[t][0][e] + acc[t][1][e];
                if (kChains == 4)
                    out[t][e] += acc[t][kChains - 2][e] + acc[t][kChains - 1][e];
            }
        const int tile_done = tile;
        tile = ntile;
        j = 0;
        if (p.independent) {
            const int n0 = tile_done * kRows + g;
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int m = 8 * t + 2 * c + (e & 1);
                    const int n = n0 + 8 * (e >> 1);
                    if (p.swiglu) {   // lane holds gate (row g) and up (row g + 8) of output 8 tile + g
                        if (e < 2 && m < p.M && n < p.N)
                            p.Y[(int64_t)m * (p.N / 2) + tile_done * 8 + g] =
                                __float2half_rn(silu(out[t][e]) * out[t][e + 2]);
                        continue;
                    }
                    if (m < p.M && n < p.N) {
                        const __half h = __float2half_rn(out[t][e]);
                        p.Y[(int64_t)m * p.N + n] = h;
                        if (kArgmax && p.argmax)   // rows ascend within a lane: '>' keeps the first maximum
                            if (__half2float(h) > best_v[t][e & 1]) {
                                best_v[t][e & 1] = __half2float(h);
                                best_i[t][e & 1] = n;
                            }
                    }
                }
        } else if (p.S == 1) {
            // one CTA per tile group: the W partial sums of each output meet in a
            // shared buffer that alternates between rounds (red, part), so one
            // barrier per round suffices
            float *rb = (r & 1) ? part : red;
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const int m0 = 8 * t + 2 * c;
                rb[(warp * kRows + g) * MP + m0] = out[t][0];
                rb[(warp * kRows + g) * MP + m0 + 1] = out[t][1];
                rb[(warp * kRows + g + 8) * MP + m0] = out[t][2];
                rb[(warp * kRows + g + 8) * MP + m0 + 1] = out[t][3];
            }
            __syncthreads();
            for (int idx = tid; idx < TPC * kRows * MP; idx += kThreads) {
                const int sl = idx / (kRows * MP), jj = idx - sl * kRows * MP;
                const int row = jj / MP, m = jj - row * MP;
                const int tl = (r * p.nclusters + cluster) * TPC + sl;
                const int n = tl * kRows + row;
                if (m >= p.M || n >= p.N || (p.swiglu && row >= 8))
                    continue;
                const float *src = rb + (sl * W * kRows) * MP + jj;
                float v = 0.f;
                for (int q = 0; q < W; q++)
                    v += src[q * kRows * MP];
                if (p.swiglu) {   // row < 8: the gate; row + 8: its up
                    float u = 0.f;
                    for (int q = 0; q < W; q++)
                        u += src[q * kRows * MP + 8 * MP];
                    p.Y[(int64_t)m * (p.N / 2) + tl * 8 + row] = __float2half_rn(silu(v) * u);
                    continue;
                }
                p.Y[(int64_t)m * p.N + n] = __float2half_rn(v);
            }
        } else {
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const int m0 = 8 * t + 2 * c;
                red[(warp * kRows + g) * MP + m0] = out[t][0];
                red[(warp * kRows + g) * MP + m0 + 1] = out[t][1];
                red[(warp * kRows + g + 8) * MP + m0] = out[t][2];
                red[(warp * kRows + g + 8) * MP + m0 + 1] = out[t][3];
            }
            __syncthreads();
            for (int idx = tid; idx < TPC * kRows * MP; idx += kThreads) {
                const int sl = idx / (kRows * MP), jj = idx - sl * kRows * MP;
                float v = 0.f;
                for (int q = 0; q < W; q++)
                    v += red[((sl * W + q) * kRows) * MP + jj];
                part[idx] = v;
            }
            if (p.S > 1) cluster_sync(); else __syncthreads();
            if (rank == 0) {
                for (int idx = tid; idx < TPC * kRows * MP; idx += kThreads) {
                    const int sl = idx / (kRows * MP), jj = idx - sl * kRows * MP;
                    const int row = jj / MP, m = jj - row * MP;
                    const int tl = (r * p.nclusters + cluster) * TPC + sl;
                    const int n = tl * kRows + row;
                    if (m >= p.M || n >= p.N || (p.swiglu && row >= 8))
                        continue;
                    float v = part[idx];
                    for (int q = 1; q < p.S; q++)
                        v += ld_dsmem_f32(part + idx, (uint32_t)q);
                    if (p.swiglu) {   // row < 8: the gate; row + 8: its up
                        float u = part[idx + 8 * MP];
                        for (int q = 1; q < p.S; q++)
                            u += ld_dsmem_f32(part + idx + 8 * MP, (uint32_t)q);
                        p.Y[(int64_t)m * (p.N / 2) + tl * 8 + row] = __float2half_rn(silu(v) * u);
                        continue;
                    }
                    p.Y[(int64_t)m * p.N + n] = __float2half_rn(v);
                }
            }
            if (p.S > 1) cluster_sync(); else __syncthreads();
        }
        ++r;
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
            for (int e = 0; e < 4 * kChains; e++) acc[t][e >> 2][e & 3] = 0.f;
    }

    if (kArgmax && p.argmax)
        argmax_finish<NT>(p, best_v, best_i, reinterpret_cast<uint2 *>(red), warp, lane, g, c, tid);

    // every issued box was waited for above; after a timeout, let the copies
    // still in flight land before the CTA's shared memory is released
    if (dead && lane == 0) {
        for (int q = (total > kDepth ? total - kDepth : 0); q < total; q++) {
            const uint32_t bar = my_bars + 8 * (q % kDepth);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(bar, (uint32_t)((q / kDepth) & 1)) && globaltimer() - t0 < kWaitLimitNs) {
            }
        }
    }
}

template <int NT, class C>
int launch_tc(const CUtensorMap &map, const TcParams &p, int grid, size_t smem, unsigned flags, cudaStream_t s) {
    auto fn = gemv_tc_kernel<NT, C>;
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, map, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

}  // namespace

// Tuning hook state: a forced K split (0 = the planner decides).
static int g_force_w = 0, g_force_s = 1;

// Shared by mnb_gemv (am == nullptr) and mnb_gemv_argmax.
static int launch_tc_common(const void *X, const uint8_t *packed, const void *scales, int scale_f16,
                            const uint8_t *zp, void *Y, int M, int N, int K, int bs, unsigned flags,
                            cudaStream_t s, const ArgmaxArgs *am, int swiglu = 0) {
    EncodeTiledFn encode = tensor_map_encoder();
    if (!encode)
        return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled unavailable");
    const int NT = (M <= 8) ? 1 : (M <= 16) ? 2 : 4;   // MMA column groups of 8 tokens
    const int MP = 8 * NT;
    const int sms = device_sm_count();

    TcParams p;
    p.X = X; p.scales = scales; p.zp = zp; p.Y = reinterpret_cast<__half *>(Y);
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.scale_f16 = scale_f16;
    p.scale_pair = (scale_f16 && bs == 32 && (p.nb % 2) == 0 && (reinterpret_cast<uintptr_t>(scales) % 4) == 0);
    p.ntiles = (N + kRows - 1) / kRows;
    p.swiglu = swiglu;
    p.argmax = am ? 1 : 0;
    p.ids = am ? am->ids : nullptr;
    p.max_out = am ? am->max_out : nullptr;
    p.ws_part = am ? reinterpret_cast<uint2 *>(static_cast<unsigned char *>(am->workspace) + kArgmaxWsHeader) : nullptr;
    p.ws_count = am ? static_cast<unsigned *>(am->workspace) : nullptr;

    // K split: W warps x S clustered CTAs per 16-row tile.  Each candidate is
    // costed in box-times on the busiest warp: rounds of tile groups x (boxes
    // per warp + a per-round reduction cost: none when warps own whole rows,
    // more when the partial sums meet across a cluster).  Fitted on the
    // decoder shapes at M <= 8 (one MMA column group); with more column groups
    // a box costs proportionally more and a cluster reduction grows with the
    // cluster (measured at two groups: 3 box-times per CTA of the cluster).
    // Four column groups take the registers of two CTAs: one CTA per SM.
    const int nbx_all = (K + kBoxK - 1) / kBoxK;
    auto smem_for = [&](int W, int S, int &nbx_w, int &kcta, int &xs_stride) {
        nbx_w = (nbx_all + W * S - 1) / (W * S);
        kcta = W * nbx_w * kBoxK;
        xs_stride = (kcta / kBoxK) * 512 + 64;
        return 1024 + (size_t)kWarps * kDepth * kBoxBytes + (size_t)M * xs_stride + 512 +
               (size_t)2 * kWarps * kRows * MP * 4 + (size_t)kWarps * kDepth * 8;
    };
    const double groups_f = (double)NT;   // MMA column groups of 8 tokens
    int W = 0, S = 1;
    double best = 0.0;
    for (int w = 1; w <= kWarps; w *= 2)
        for (int sc = 1; sc <= kMaxCluster; sc *= 2) {
            if ((w * sc > nbx_all && !(w == 1 && sc == 1)) || (am && (w != 1 || sc != 1)))
                continue;
            int nbx_w, kcta, xs_stride;
            const size_t sm_ = smem_for(w, sc, nbx_w, kcta, xs_stride);
            if (sm_ > 200 * 1024)
                continue;
            const int per_sm = (NT < 4 && sm_ <= 110 * 1024) ? 2 : 1;
            double cost;
            if (w == 1 && sc == 1) {
                const int warps = sms * per_sm * kWarps;
                cost = (double)((p.ntiles + warps - 1) / warps) * nbx_all * groups_f;
            } else {
                const int tpc = kWarps / w;
                const int groups = (p.ntiles + tpc - 1) / tpc;
                int maxcl = sms * per_sm / sc;
                if (maxcl < 1) maxcl = 1;
                const int rounds = (groups + maxcl - 1) / maxcl;
                const double red = (sc == 1) ? 0.5 * groups_f : (NT == 1 ? 1.6 : 1.5 * groups_f * sc);
                cost = rounds * (1.15 * groups_f * nbx_w + red);
            }
            if (W == 0 || cost < best - 1e-9 || (cost < best + 1e-9 && sc < S) ||
                (cost < best + 1e-9 && sc == S && w > W)) {
                W = w;
                S = sc;
                best = cost;
            }
        }
    if (!am && g_force_w > 0) {   // tuning hook
        W = g_force_w;
        S = g_force_s;
    }
    if (W == 0)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: K=%d too large for M=%d", K, M);
    size_t smem = 0;
    {
        int nbx_w, kcta, xs_stride;
        smem = smem_for(W, S, nbx_w, kcta, xs_stride);
        p.S = S; p.W = W; p.nbx_w = nbx_w; p.kcta = kcta; p.xs_stride = xs_stride;
    }
    if (smem > 220 * 1024)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: K=%d too large for M=%d", K, M);
    p.independent = (p.W == 1 && p.S == 1);
    const int per_sm = (NT < 4 && smem <= 110 * 1024) ? 2 : 1;
    int grid;
    if (p.independent) {
        const int groups = (p.ntiles + kWarps - 1) / kWarps;
        grid = groups < sms * per_sm ? groups : sms * per_sm;
        p.rounds = 0;
        p.nclusters = grid;
    } else {
        const int tpc = kWarps / p.W;
        const int groups = (p.ntiles + tpc - 1) / tpc;
        int max_clusters = sms * per_sm / p.S;
        if (max_clusters < 1) max_clusters = 1;
        p.rounds = (groups + max_clusters - 1) / max_clusters;
        p.nclusters = (groups + p.rounds - 1) / p.rounds;
        grid = p.nclusters * p.S;
    }

    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
    const cuuint64_t gstride[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {128, (cuuint32_t)kRows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS)
        return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled failed (%d)", (int)cr);
    // fp16 scales read as aligned pairs (block 32) or singly (block 64)
    const bool fast_scales = scale_f16 && (bs == 64 || p.scale_pair);
    const bool bs64 = (bs == 64), has_zp = (zp != nullptr);
#define MNB_TC(NT_, B_, Z_, S_) return launch_tc<NT_, Cfg<B_, Z_, S_>>(map, p, grid, smem, flags, s)
#define MNB_TC_S(NT_, B_, Z_) \
    if (fast_scales) MNB_TC(NT_, B_, Z_, 0); else MNB_TC(NT_, B_, Z_, 1)
#define MNB_TC_Z(NT_, B_) \
    if (has_zp) { MNB_TC_S(NT_, B_, true); } else { MNB_TC_S(NT_, B_, false); }
    if (NT == 1) {
        if (bs64) { MNB_TC_Z(1, true); } else { MNB_TC_Z(1, false); }
    } else if (NT == 2) {
        if (bs64) { MNB_TC_Z(2, true); } else { MNB_TC_Z(2, false); }
    } else {
        if (bs64) { MNB_TC_Z(4, true); } else { MNB_TC_Z(4, false); }
    }
#undef MNB_TC_Z
#undef MNB_TC_S
#undef MNB_TC
}

int launch_gemv_tc(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                   void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s) {
    return launch_tc_common(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s, nullptr);
}

int launch_gemv_swiglu(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                       void *Y, int M, int N, int K, int bs, unsigned flags, cudaStream_t s) {
    if (M == 1 && scale_f16 && gemv_resident_enabled()) {   // the one-token kernel, as mnb_gemv at M = 1
        const int rc = launch_gemv_resident(X, packed, scales, zp, Y, N, K, bs, flags, s, nullptr, nullptr, nullptr, 1);
        if (rc != 1)
            return rc;
    }
    return launch_tc_common(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s, nullptr, 1);
}

size_t gemv_argmax_workspace_bytes(int M) {
    // one (value, index) pair per token per CTA; at most two CTAs per SM
    return kArgmaxWsHeader + (size_t)2 * device_sm_count() * (size_t)M * sizeof(uint2);
}

int launch_gemv_argmax(const void *X, const uint8_t *packed, const void *scales, int scale_f16, const uint8_t *zp,
                       void *Y, int M, int N, int K, int bs, int32_t *ids, float *max_out, void *workspace,
                       unsigned flags, cudaStream_t s) {
    if (M == 1 && scale_f16 && gemv_resident_enabled()) {   // the one-token kernel, as mnb_gemv at M = 1
        const int rc = launch_gemv_resident(X, packed, scales, zp, Y, N, K, bs, flags, s, ids, max_out, workspace);
        if (rc != 1)
            return rc;
    }
    ArgmaxArgs am{ids, max_out, workspace};
    return launch_tc_common(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s, &am);
}

// ---- greedy decoding without a caller-provided workspace -------------------
//
// The scratch of mnb_gemv_argmax_noalloc lives in this module-scope device
// array: every GPU that loads the library holds these 64 KiB until the process
// exits, and every call on that GPU shares them.  Host code must not hand the
// array's name to a kernel (on the host it is only a stand-in for the symbol):
// the first call on each device asks the runtime for the array's device
// address, with that device current, and later calls reuse it.
constexpr size_t kNoAllocScratchBytes = 64 * 1024;
static __device__ __align__(256) unsigned char g_argmax_scratch[kNoAllocScratchBytes];

static int noalloc_scratch_ptr(void **out) {
    static std::mutex mu;
    static void *ptrs[128] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv_argmax_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 128)
        return fail(MNB_ERR_UNSUPPORTED, "mnb_gemv_argmax_noalloc: device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_argmax_scratch);
        if (e != cudaSuccess || !p)
            return fail(MNB_ERR_CUDA, "mnb_gemv_argmax_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return MNB_OK;
}

size_t gemv_argmax_noalloc_capacity() { return kNoAllocScratchBytes; }

int launch_gemv_argmax_noalloc(const void *X, const uint8_t *packed, const void *scales, int scale_f16,
                               const uint8_t *zp, void *Y, int M, int N, int K, int bs, int32_t *ids,
                               float *max_out, unsigned flags, cudaStream_t s) {
    const size_t need = gemv_argmax_workspace_bytes(M);
    if (need > kNoAllocScratchBytes)
        return fail(MNB_ERR_SHAPE, "mnb_gemv_argmax_noalloc: M=%d needs %zu bytes of scratch, the library holds %zu",
                    M, need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    int rc = noalloc_scratch_ptr(&scratch);
    if (rc)
        return rc;
    // the CTA counter must start at zero; a call cut short could have left it set
    cudaError_t e = cudaMemsetAsync(scratch, 0, kArgmaxWsHeader, s);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv_argmax_noalloc: clearing the scratch counter: %s", cudaGetErrorString(e));
    return launch_gemv_argmax(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, ids, max_out, scratch, flags, s);
}

int read_gemv_status(unsigned *out, int clear) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_gemv_status, sizeof(unsigned));
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_gemv_status, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_device_status: %s", cudaGetErrorString(e));
    *out |= v;
    return MNB_OK;
}

}  // namespace mnb

// Tuning hook: force the decode kernel's K split to W warps x S clustered CTAs
// per 16-row tile (w = 0 restores the planner).  Not part of the stable ABI.
extern "C" MNB_API int mnb_tune_gemv_split(int w, int s) {
    if (w < 0 || w > 8 || (w & (w - 1)) != 0 || s < 1 || s > 8)
        return MNB_ERR_INVALID_ARG;
    mnb::g_force_w = w;
    mnb::g_force_s = s;
    return MNB_OK;
}
