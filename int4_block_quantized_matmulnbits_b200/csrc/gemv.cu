// gemv.cu -- decode-shaped MatMulNBits with fp32 activations (the q4 variant of
// "Qwen3-ASR-0.6B -- ONNX for the browser", "Pick a variant"):
// Y[M][N] = X[M][K] . dequant(W)^T with 1 <= M <= 16 (the per-token
// decoder_step of the same page, "Graph contracts").  fp16 activations go to
// gemv_tc.cu.
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
// Unpack + dequant happen in registers: (0x4B000000 | q) is the fp32 2^23 + q
// exactly, so subtracting 2^23 + zp leaves the exact q - zp.  The inner product
// takes true fp32 FMAs (the fp32 tolerance leaves no room for fp16 products):
// an fp32 partial per 32-k chunk, times the scale, summed in fp32, reduced
// across the 4 lanes of a row with warp shuffles.
#include "common.cuh"
#include "internal.h"
#include "mnb_tune.h"

namespace mnb {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;
constexpr int kPF = 4;            // super-chunks in flight per warp
constexpr int kSuper = 128;       // k per super-chunk
constexpr int kMaxCluster = 8;


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
    float s0, s1;      // scales as fp32
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
// Scales are delivered as fp32 (an fp16 scale converts exactly).
__device__ __forceinline__ Slot load_advance(const Params &p, Cursor &q, bool live, int zsh,
                                             int tile_step_base, int g, int kfirst) {
    Slot s;
    s.p0 = s.p1 = make_uint4(0, 0, 0, 0);
    s.s0 = s.s1 = 0.f;
    s.z0 = s.z1 = 8;
    if (live && q.k < p.K) {
#pragma unroll
        for (int r = 0; r < 2; r++) {
            if (!(r ? q.ok1 : q.ok0))
                continue;
            const int64_t rows8 = r ? 8 : 0;
            const uint4 v = ldg_stream_v4(q.p0 + rows8 * (p.K / 2));
            const uint8_t *sp = q.s0 + rows8 * p.nb * (p.scale_f16 ? 2 : 4);
            const float sb = p.scale_f16
                                 ? __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(sp))))
                                 : __ldg(reinterpret_cast<const float *>(sp));
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

__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }



__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// MP: tokens held per thread (1, 2, 4, 8 or 16).
template <int MP>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
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
        ring[i] = load_advance(p, cur_ld, i < total, zsh, tile_base, g, kfirst);
    pdl_launch_dependents();
    pdl_wait();

    // ---- stage X[0:M, kcta0 : kcta0 + kcta), zero past K
    const int nsc_cta = W * p.nsc_w;
    {
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

    float acc[2][MP];   // rows g, g+8 x tokens
#pragma unroll
    for (int r = 0; r < 2; r++)
#pragma unroll
        for (int m = 0; m < MP; m++) acc[r][m] = 0.f;

    int cr = 0, csc = 0;   // position being consumed
    for (int base = 0; base < total; base += kPF) {
#pragma unroll
        for (int i = 0; i < kPF; i++) {
            if (base + i >= total)
                break;
            const Slot cur = ring[i];
            ring[i] = load_advance(p, cur_ld, base + i + kPF < total, zsh, tile_base, g, kfirst);
            const int sc = wk * p.nsc_w + csc;   // super-chunk inside the CTA's X range

            // exact (q - zp) as fp32 via 2^23 + q
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
                const unsigned char *xa = xs + m * p.xs_stride + sc * 512 + c * 16;
                float pa = 0.f, pb = 0.f;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint4 v = lds128(xa + j * 64);
                    const float xv[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                                         __uint_as_float(v.w)};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        pa = fmaf(xv[e], fa[4 * j + e], pa);
                        pb = fmaf(xv[e], fb[4 * j + e], pb);
                    }
                }
                acc[0][m] = fmaf(cur.s0, pa, acc[0][m]);
                acc[1][m] = fmaf(cur.s1, pb, acc[1][m]);
            }

            if (++csc < p.nsc_w)
                continue;
            // ---- end of this round's tile for every warp of the CTA (uniform)
            csc = 0;
            const int r = cr++;
#pragma unroll
            for (int rr = 0; rr < 2; rr++)
#pragma unroll
                for (int m = 0; m < MP; m++) {
                    acc[rr][m] += __shfl_xor_sync(0xffffffffu, acc[rr][m], 1);
                    acc[rr][m] += __shfl_xor_sync(0xffffffffu, acc[rr][m], 2);
                }
            float *Y = reinterpret_cast<float *>(p.Y);
            if (W == 1 && p.S == 1) {
                // the warp holds the whole dot product: write Y straight from registers
                const int n0 = tile_at(r, slot) * kRows + g;
                if (c == 0) {
#pragma unroll
                    for (int rr = 0; rr < 2; rr++)
#pragma unroll
                        for (int m = 0; m < MP; m++) {
                            const int n = n0 + 8 * rr;
                            if (m < p.M && n < p.N)
                                Y[(int64_t)m * p.N + n] = acc[rr][m];
                        }
                }
            } else {
                // partials: warps of a tile in shared memory, then CTAs of the cluster
                if (c == 0) {
#pragma unroll
                    for (int rr = 0; rr < 2; rr++)
#pragma unroll
                        for (int m = 0; m < MP; m++)
                            red[(warp * kRows + g + 8 * rr) * MP + m] = acc[rr][m];
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
                        Y[(int64_t)m * p.N + n] = v;
                    }
                }
                if (p.S > 1) cluster_sync(); else __syncthreads();
            }
#pragma unroll
            for (int rr = 0; rr < 2; rr++)
#pragma unroll
                for (int m = 0; m < MP; m++) acc[rr][m] = 0.f;
        }
    }
}

template <int MP>
int launch_one(const Params &p, int grid, size_t smem, unsigned flags, cudaStream_t s) {
    auto fn = gemv_kernel<MP>;
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

// Work decomposition: K slices = W warps x S CTAs per tile, chosen so that
// about two CTAs of 8 warps per SM have work; rounds of tiles per CTA, with the
// CTA count balanced so every CTA walks the same number of rounds.
static int plan_gemv(int M, int N, int K, int MP, int sms, Params &p, int &grid, size_t &smem) {
    const int esz = 4;   // fp32 activations
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

// One-token fp16 calls go to the resident kernel (1) or the general one (0).
static int g_resident = 1;

int gemv_resident_enabled() { return g_resident; }

int launch_gemv(const void *X, int act_f16, const uint8_t *packed, const void *scales,
                int scale_f16, const uint8_t *zp, void *Y, int M, int N, int K, int bs,
                unsigned flags, cudaStream_t s) {
    if (act_f16) {   // tensor-core paths, weights moved by TMA
        if (M == 1 && scale_f16 && g_resident) {
            const int rc = launch_gemv_resident(X, packed, scales, zp, Y, N, K, bs, flags, s);
            if (rc != 1)
                return rc;
        }
        return launch_gemv_tc(X, packed, scales, scale_f16, zp, Y, M, N, K, bs, flags, s);
    }
    const int MP = (M <= 1) ? 1 : (M <= 2) ? 2 : (M <= 4) ? 4 : (M <= 8) ? 8 : 16;

    Params p;
    p.X = X; p.packed = packed; p.scales = scales; p.zp = zp; p.Y = Y;
    p.M = M; p.N = N; p.K = K;
    p.bs_shift = (bs == 64) ? 1 : 0;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.scale_f16 = scale_f16;
    int grid = 0;
    size_t smem = 0;
    int rc = plan_gemv(M, N, K, MP, device_sm_count(), p, grid, smem);
    if (rc)
        return rc;
    switch (MP) {
        case 1: return launch_one<1>(p, grid, smem, flags, s);
        case 2: return launch_one<2>(p, grid, smem, flags, s);
        case 4: return launch_one<4>(p, grid, smem, flags, s);
        case 8: return launch_one<8>(p, grid, smem, flags, s);
        default: return launch_one<16>(p, grid, smem, flags, s);
    }
}

}  // namespace mnb

// Tuning hook: 1 (default) sends one-token fp16 GEMVs to the resident decode
// kernel where it applies, 0 to the general decode kernel.  Declared in
// mnb_tune.h.
extern "C" MNB_API int mnb_tune_gemv_resident(int enable) {
    if (enable != 0 && enable != 1)
        return MNB_ERR_INVALID_ARG;
    mnb::g_resident = enable;
    return MNB_OK;
}
