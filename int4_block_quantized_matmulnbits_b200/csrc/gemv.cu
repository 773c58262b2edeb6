// gemv.cu -- decode-shaped MatMulNBits, Y[M][N] = X[M][K] . dequant(W)^T with
// 1 <= M <= 16 (the per-token decoder_step of "Qwen3-ASR-0.6B -- ONNX for the
// browser", "Graph contracts", and of "Mega-ASR -- INT4 ONNX", "What's in this
// repo": decoder_step_int4).
//
// This is HBM-bound: every packed byte is read exactly once, so the kernel is
// built around moving weight bytes.
//   * A warp owns a tile of 16 weight rows over a K slice.  Thread (g = lane/4,
//     c = lane%4) owns rows g and g+8; the warp walks "super-chunks" of 128 k,
//     in which thread c loads the 16-byte chunk c (32 nibbles, one block of 32
//     or half a block of 64) of both rows with 128-bit streaming loads.  The
//     warp's four loads of a row are one contiguous 64-byte segment.
//   * CTAs (8 warps) are persistent: the grid is sized to the SMs and every
//     CTA walks rounds of tiles, so X is staged in shared memory once per CTA
//     and the weight prefetch ring runs straight across tile boundaries.
//   * Weights are prefetched into a register ring several super-chunks deep,
//     and the first loads are issued BEFORE griddepcontrol.wait, so under
//     programmatic dependent launch the weight stream of this kernel overlaps
//     the tail of the previous one; X is read only after the wait.
//   * When the row tiles alone cannot occupy the SMs, K is split, first over
//     W warps of the CTA (partials meet in shared memory), then over a
//     thread-block cluster of S CTAs (partials meet in distributed shared
//     memory): no global scratch, no second kernel, no atomics.
//   * X for the CTA's K range is staged permuted, so one 16-byte load yields
//     the activation pairs that match the dequantized weight pairs.
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

constexpr int kWarps = 8;
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
    int S;          // CTAs per cluster (K split across CTAs)
    int W;          // warps per tile inside a CTA (K split across warps); divides kWarps
    int nsc_w;      // super-chunks of one warp's K slice
    int kcta;       // k covered by one CTA = W * nsc_w * kSuper
    int rounds;     // tile rounds per CTA
    int nclusters;  // gridDim.x / S
    int xs_stride;  // bytes per token row of the staged X
};

struct Slot {
    uint4 p0, p1;      // 32 nibbles of row g and of row g+8
    uint32_t s0, s1;   // scales, already in the inner product's type: fp16 bits
                       // (tensor-core path) or fp32 bits (CUDA-core path)
    uint32_t z0, z1;   // zero point nibble (8 when absent)
};

// A thread's streaming position in its warp's sequence of (round, super-chunk):
// pointers to its 16-byte chunk of rows g and g+8 and to that chunk's scale and
// zero-point byte.  Moving to the next super-chunk is a few pointer additions;
// only a change of tile recomputes them.
struct Cursor {
    const uint8_t *p0;        // packed bytes of row g (row g+8 is 8 rows further)
    const uint8_t *s0;        // its scale (fp16 or fp32 bytes)
    const uint8_t *z0;        // its zero-point byte
    int k;                    // first k of the thread's chunk
    int sc, r;                // super-chunk in the slice, round
    bool ok0, ok1;            // row g / g+8 inside N
};

__device__ __forceinline__ void cursor_tile(const Params &p, Cursor &q, int tile, int g, int kfirst) {
    const int n0 = tile * kRows + g, ssz = p.scale_f16 ? 2 : 4;
    const int blk = kfirst >> (5 + p.bs_shift);
    q.k = kfirst;
    q.ok0 = n0 < p.N;
    q.ok1 = n0 + 8 < p.N;
    q.p0 = p.packed + (int64_t)n0 * (p.K / 2) + kfirst / 2;
    q.s0 = reinterpret_cast<const uint8_t *>(p.scales) + ((int64_t)n0 * p.nb + blk) * ssz;
    q.z0 = p.zp ? p.zp + (int64_t)n0 * p.zpb + (blk >> 1) : nullptr;
}

// Loads the cursor's super-chunk (nothing when !live or past K), then advances.
// SCALE_F16: deliver the scales as fp16 bits (an fp32 scale is rounded once,
// here); else as fp32 bits.
template <bool SCALE_F16>
__device__ __forceinline__ Slot load_advance(const Params &p, Cursor &q, bool live, int zsh,
                                             int tile_step_base, int g, int kfirst) {
    Slot s;
    s.p0 = s.p1 = make_uint4(0, 0, 0, 0);
    s.s0 = s.s1 = 0;
    s.z0 = s.z1 = 8;
    if (live && q.k < p.K) {
#pragma unroll
        for (int r = 0; r < 2; r++) {
            if (!(r ? q.ok1 : q.ok0))
                continue;
            const int64_t rows8 = r ? 8 : 0;
            const uint4 v = ldg_stream_v4(q.p0 + rows8 * (p.K / 2));
            const uint8_t *sp = q.s0 + rows8 * p.nb * (p.scale_f16 ? 2 : 4);
            uint32_t sb;
            if (p.scale_f16) {
                const unsigned short h = __ldg(reinterpret_cast<const unsigned short *>(sp));
                sb = SCALE_F16 ? (uint32_t)h : __float_as_uint(__half2float(__ushort_as_half(h)));
            } else {
                const float f = __ldg(reinterpret_cast<const float *>(sp));
                sb = SCALE_F16 ? (uint32_t)__half_as_ushort(__float2half_rn(f)) : __float_as_uint(f);
            }
            uint32_t z = 8;
            if (p.zp)
                z = ((uint32_t)__ldg(q.z0 + rows8 * p.zpb) >> zsh) & 15u;
            if (r == 0) { s.p0 = v; s.s0 = sb; s.z0 = z; }
            else        { s.p1 = v; s.s1 = sb; s.z1 = z; }
        }
    }
    // next super-chunk: 64 packed bytes, 128 / bs blocks further
    const int ssz = p.scale_f16 ? 2 : 4;
    const int bstep = 4 >> p.bs_shift;
    q.p0 += 64;
    q.s0 += bstep * ssz;
    if (p.zp) q.z0 += bstep >> 1;
    q.k += kSuper;
    if (++q.sc == p.nsc_w) {
        q.sc = 0;
        ++q.r;
        cursor_tile(p, q, (q.r * p.nclusters) * (kWarps / p.W) + tile_step_base, g, kfirst);
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

__device__ __forceinline__ half2 scale_h2(uint32_t h16) { return u32_as_h2(h16 | (h16 << 16)); }

__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }



__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// MP: tokens held per thread (MMA: 8 or 16, CC: 1, 2, 4, 8 or 16).
template <int MODE, bool ACT_F16, int MP>
__global__ void __launch_bounds__(kThreads, (MODE == MODE_MMA) ? 2 : 1) gemv_kernel(const Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NT = (MODE == MODE_MMA) ? MP / 8 : 1;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int W = p.W, TPC = kWarps / p.W;
    const int slot = warp / W, wk = warp - slot * W;
    const int rank = (p.S > 1) ? (int)cluster_ctarank() : 0;
    const int cluster = blockIdx.x / p.S;
    const int kcta0 = rank * p.kcta;                   // first k of this CTA
    const int kw = kcta0 + wk * p.nsc_w * kSuper;      // first k of this warp's slice
    const int total = p.rounds * p.nsc_w;              // super-chunks this warp walks

    unsigned char *xs = smem;                                              // [M][xs_stride]
    float *red = reinterpret_cast<float *>(smem + p.M * p.xs_stride);      // [kWarps][16][MP]
    float *part = red + kWarps * kRows * MP;                                // [TPC][16][MP]
    // tile handled by slot `sl` of this CTA in round r
    auto tile_at = [&](int r, int sl) { return (r * p.nclusters + cluster) * TPC + sl; };

    // ---- weights first: they do not depend on the previous kernel
    const int kfirst = kw + c * 32;
    const int zsh = 4 * ((kfirst >> (5 + p.bs_shift)) & 1);   // nibble of this thread's blocks
    const int tile_base = cluster * TPC + slot;                  // tile in round r: r * nclusters * TPC + base
    Cursor cur_ld;
    cur_ld.sc = 0;
    cur_ld.r = 0;
    cursor_tile(p, cur_ld, tile_base, g, kfirst);
    Slot ring[kPF];
#pragma unroll
    for (int i = 0; i < kPF; i++)
        ring[i] = load_advance<MODE == MODE_MMA>(p, cur_ld, i < total, zsh, tile_base, g, kfirst);
    pdl_launch_dependents();
    pdl_wait();

    // ---- stage X[0:M, kcta0 : kcta0 + kcta), zero past K
    const int nsc_cta = W * p.nsc_w;
    if (ACT_F16) {
        const __half *X = reinterpret_cast<const __half *>(p.X);
        const int per_tok = nsc_cta * 16;                      // 16-byte units of 8 halves
        for (int u = tid; u < p.M * per_tok; u += kThreads) {
            const int m = u / per_tok;
            const int r = u - m * per_tok;
            const int sc = r >> 4, cc = (r >> 2) & 3, w = r & 3;
            const int k = kcta0 + sc * kSuper + cc * 32 + w * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (k < p.K)
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
        const int per_tok = nsc_cta * 32;                      // 16-byte units of 4 floats
        for (int u = tid; u < p.M * per_tok; u += kThreads) {
            const int m = u / per_tok;
            const int r = u - m * per_tok;
            const int sc = r >> 5, cc = (r >> 3) & 3, j = r & 7;
            const int k = kcta0 + sc * kSuper + cc * 32 + j * 4;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (k < p.K)
                v = ldg_v4(X + (int64_t)m * p.K + k);
            *reinterpret_cast<uint4 *>(xs + m * p.xs_stride + sc * 512 + j * 64 + cc * 16) = v;
        }
    }
    __syncthreads();

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

    const unsigned char *xs_base = xs;
    int cr = 0, csc = 0;   // position being consumed
    for (int base = 0; base < total; base += kPF) {
#pragma unroll
        for (int i = 0; i < kPF; i++) {
            if (base + i >= total)
                break;
            const Slot cur = ring[i];
            ring[i] = load_advance<MODE == MODE_MMA>(p, cur_ld, base + i + kPF < total, zsh, tile_base, g,
                                                       kfirst);
            const int sc = wk * p.nsc_w + csc;   // super-chunk inside the CTA's X range

            if (MODE == MODE_MMA) {
                uint32_t wa[16], wb[16];
                dq_chunk(cur.p0, cur.z0, wa);
                dq_chunk(cur.p1, cur.z1, wb);
                const half2 s0 = scale_h2(cur.s0);
                const half2 s1 = scale_h2(cur.s1);
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    wa[j] = h2_as_u32(__hmul2(u32_as_h2(wa[j]), s0));
                    wb[j] = h2_as_u32(__hmul2(u32_as_h2(wb[j]), s1));
                }
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    uint32_t xb[16];
                    const int tok = g + 8 * t;
                    if (tok < p.M) {
                        const unsigned char *xa = xs_base + tok * p.xs_stride + sc * 256 + c * 16;
#pragma unroll
                        for (int w = 0; w < 4; w++) {
                            const uint4 v = lds128(xa + w * 64);
                            xb[4 * w + 0] = v.x; xb[4 * w + 1] = v.y;
                            xb[4 * w + 2] = v.z; xb[4 * w + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; j++) xb[j] = 0u;
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
                const float s0 = __uint_as_float(cur.s0);
                const float s1 = __uint_as_float(cur.s1);
#pragma unroll
                for (int m = 0; m < MP; m++) {
                    if (m >= p.M)
                        break;
                    const unsigned char *xa = xs_base + m * p.xs_stride + sc * 256 + c * 16;
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
                const float s0 = __uint_as_float(cur.s0);
                const float s1 = __uint_as_float(cur.s1);
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
                    if (m >= p.M)
                        break;
                    const unsigned char *xa = xs_base + m * p.xs_stride + sc * 512 + c * 16;
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

            if (++csc < p.nsc_w)
                continue;
            // ---- end of this round's tile for every warp of the CTA (uniform)
            csc = 0;
            const int r = cr++;
            if (MODE == MODE_CC) {
#pragma unroll
                for (int rr = 0; rr < 2; rr++)
#pragma unroll
                    for (int m = 0; m < MP; m++) {
                        accc[rr][m] += __shfl_xor_sync(0xffffffffu, accc[rr][m], 1);
                        accc[rr][m] += __shfl_xor_sync(0xffffffffu, accc[rr][m], 2);
                    }
            }
            if (W == 1 && p.S == 1) {
                // the warp holds the whole dot product: write Y straight from registers
                const int n0 = tile_at(r, slot) * kRows + g;
                if (MODE == MODE_MMA) {
#pragma unroll
                    for (int t = 0; t < NT; t++)
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const int m = 8 * t + 2 * c + (e & 1);
                            const int n = n0 + 8 * (e >> 1);
                            if (m < p.M && n < p.N)
                                reinterpret_cast<__half *>(p.Y)[(int64_t)m * p.N + n] = __float2half_rn(accm[t][e]);
                        }
                } else if (c == 0) {
#pragma unroll
                    for (int rr = 0; rr < 2; rr++)
#pragma unroll
                        for (int m = 0; m < MP; m++) {
                            const int n = n0 + 8 * rr;
                            if (m < p.M && n < p.N) {
                                if (ACT_F16)
                                    reinterpret_cast<__half *>(p.Y)[(int64_t)m * p.N + n] = __float2half_rn(accc[rr][m]);
                                else
                                    reinterpret_cast<float *>(p.Y)[(int64_t)m * p.N + n] = accc[rr][m];
                            }
                        }
                }
            } else {
                // partials: warps of a tile in shared memory, then CTAs of the cluster
                if (MODE == MODE_MMA) {
#pragma unroll
                    for (int t = 0; t < NT; t++) {
                        const int m0 = 8 * t + 2 * c;
                        red[(warp * kRows + g) * MP + m0] = accm[t][0];
                        red[(warp * kRows + g) * MP + m0 + 1] = accm[t][1];
                        red[(warp * kRows + g + 8) * MP + m0] = accm[t][2];
                        red[(warp * kRows + g + 8) * MP + m0 + 1] = accm[t][3];
                    }
                } else if (c == 0) {
#pragma unroll
                    for (int rr = 0; rr < 2; rr++)
#pragma unroll
                        for (int m = 0; m < MP; m++)
                            red[(warp * kRows + g + 8 * rr) * MP + m] = accc[rr][m];
                }
                __syncthreads();
                for (int idx = tid; idx < TPC * kRows * MP; idx += kThreads) {
                    const int sl = idx / (kRows * MP), j = idx - sl * kRows * MP;
                    float v = 0.f;
                    for (int q = 0; q < W; q++)
                        v += red[((sl * W + q) * kRows) * MP + j];
                    part[idx] = v;
                }
                if (p.S > 1) cluster_sync(); else __syncthreads();
                if (rank == 0) {
                    for (int idx = tid; idx < TPC * kRows * MP; idx += kThreads) {
                        const int sl = idx / (kRows * MP), j = idx - sl * kRows * MP;
                        const int row = j / MP, m = j - row * MP;
                        const int n = tile_at(r, sl) * kRows + row;
                        if (m >= p.M || n >= p.N)
                            continue;
                        float v = part[idx];
                        for (int q = 1; q < p.S; q++)
                            v += ld_dsmem_f32(part + idx, (uint32_t)q);
                        if (ACT_F16)
                            reinterpret_cast<__half *>(p.Y)[(int64_t)m * p.N + n] = __float2half_rn(v);
                        else
                            reinterpret_cast<float *>(p.Y)[(int64_t)m * p.N + n] = v;
                    }
                }
                if (p.S > 1) cluster_sync(); else __syncthreads();
            }
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int e = 0; e < 4; e++) accm[t][e] = 0.f;
#pragma unroll
            for (int rr = 0; rr < 2; rr++)
#pragma unroll
                for (int m = 0; m < MP; m++) accc[rr][m] = 0.f;
        }
    }
}

template <int MODE, bool ACT_F16, int MP>
int launch_one(const Params &p, int grid, size_t smem, unsigned flags, cudaStream_t s) {
    auto fn = gemv_kernel<MODE, ACT_F16, MP>;
    static int configured[kMaxDevices] = {};   // largest dynamic shared memory opted into, per device
    if ((int)smem > 48 * 1024) {
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}


}  // namespace

// Which inner product serves fp16 activations at M = 1 and 2: MMA by default.
static int g_gemv_f16_cc_max_m = 0;
// 1: fp16 activations go to the warp-specialized streaming kernel for the shapes
// it serves.  Off by default: on the decoder shapes it is not yet faster than
// the general TMA kernel.
static int g_gemv_stream = 0;

// Work decomposition: K slices = W warps x S CTAs per tile, chosen so that
// about two CTAs of 8 warps per SM have work; rounds of tiles per CTA, with the
// CTA count balanced so every CTA walks the same number of rounds.
int plan_gemv(int M, int N, int K, int esz, int MP, int sms, Params &p, int &grid, size_t &smem) {
    const int tiles = (N + kRows - 1) / kRows;
    const int nsc_all = (K + kSuper - 1) / kSuper;
    const int target_warps = sms * 2 * kWarps;
    int slices = (target_warps + tiles - 1) / tiles;
    if (slices > nsc_all) slices = nsc_all;
    if (slices > kWarps * kMaxCluster) slices = kWarps * kMaxCluster;
    if (slices < 1) slices = 1;
    int W = 1;
    while (W * 2 <= kWarps && W * 2 <= slices) W *= 2;
    int S = (slices + W - 1) / W;
    if (S > kMaxCluster) S = kMaxCluster;
    for (;; S++) {
        int nsc_w = (nsc_all + W * S - 1) / (W * S);
        const int kcta = W * nsc_w * kSuper;
        const int xs_stride = nsc_w * W * kSuper * esz + 64;
        smem = (size_t)M * xs_stride + (size_t)(kWarps + kWarps) * kRows * MP * 4;
        p.S = S; p.W = W; p.nsc_w = nsc_w; p.kcta = kcta; p.xs_stride = xs_stride;
        if (smem <= 100 * 1024 || S >= kMaxCluster)
            break;
    }
    if (smem > 200 * 1024)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: K=%d too large for M=%d", K, M);
    const int tpc = kWarps / p.W;
    const int groups = (tiles + tpc - 1) / tpc;
    const int per_sm = (M * p.xs_stride > 60 * 1024) ? 1 : 2;
    int max_clusters = sms * per_sm / p.S;
    if (max_clusters < 1) max_clusters = 1;
    p.rounds = (groups + max_clusters - 1) / max_clusters;
    p.nclusters = (groups + p.rounds - 1) / p.rounds;
    if ((int64_t)p.nclusters * p.S > 0x7fffffff)
        return fail(MNB_ERR_SHAPE, "mnb_gemv: N too large");
    grid = p.nclusters * p.S;
    return MNB_OK;
}

int launch_gemv(const void *X, int act_f16, const uint8_t *packed, const void *scales,
                int scale_f16, const uint8_t *zp, void *Y, int M, int N, int K, int bs,
                unsigned flags, cudaStream_t s) {
    if (act_f16 && (M > g_gemv_f16_cc_max_m || M > 16)) {   // tensor-core paths, weights streamed by TMA
        if (g_gemv_stream) {
            const int rc = launch_gemv_stream(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s);
            if (rc != 1)
                return rc;
        }
        return launch_gemv_tc(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s);
    }
    const int mode = MODE_CC;
    int MP;
    if (mode == MODE_MMA)
        MP = (M <= 8) ? 8 : 16;
    else
        MP = (M <= 1) ? 1 : (M <= 2) ? 2 : (M <= 4) ? 4 : (M <= 8) ? 8 : 16;

    Params p;
    p.X = X; p.packed = packed; p.scales = scales; p.zp = zp; p.Y = Y;
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.scale_f16 = scale_f16;
    int grid = 0;
    size_t smem = 0;
    int rc = plan_gemv(M, N, K, act_f16 ? 2 : 4, MP, device_sm_count(), p, grid, smem);
    if (rc)
        return rc;

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

// Tuning hook: 0 (default) sends every fp16 GEMV to the general TMA kernel, 1
// lets the streaming kernel take the shapes it serves.  Not part of the stable ABI.
extern "C" MNB_API int mnb_tune_gemv_stream(int enable) {
    if (enable != 0 && enable != 1)
        return MNB_ERR_INVALID_ARG;
    mnb::g_gemv_stream = enable;
    return MNB_OK;
}
