// gemv_resident.cu -- decode-shaped MatMulNBits for ONE token with fp16
// activations: y[N] = x[K] . dequant(W)^T, the per-token decoder step of
// "Qwen3-ASR-0.6B -- ONNX for the browser" ("Graph contracts": decoder_step,
// input_embeds [1, 1, 1024]) and of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)"
// (decoder_step_int4).
//
// A decode step is a chain of ~200 such GEMVs, each waiting for the one before
// it.  Most move 1-7 MB of weights -- well under 2 us of HBM time -- so what
// costs is the critical path from "previous kernel done" to "this kernel's y
// stored".  This kernel is built to keep that path short:
//   * Half an SM per CTA (8 working warps, <= 96 registers, ~110 KB of shared
//     memory), one CTA per SM.  While kernel i runs, the CTAs of kernel i+1
//     (launched early by programmatic dependent launch) sit on the other half
//     of every SM and pull ALL of their weights into shared memory: each warp
//     owns a ring of `depth` slots, one slot = one 16-row x 256-k box of
//     packed bytes (TMA, 128-byte swizzle) plus its scales and zero points
//     (cp.async), completing on one mbarrier.  For the decoder's projections
//     every unit fits in the rings, so after griddepcontrol.wait only x is
//     read from memory.  The lm_head streams through the same rings, with
//     one 20-warp CTA per SM.
//   * Work split: CTA b owns a contiguous run of 16-row tiles; its (tile, box)
//     units are cut into one contiguous run per warp.  Tiles a warp covers
//     whole are stored from registers; the partial sums of tiles cut between
//     warps meet in shared memory and are added in warp order.  Both launch
//     shapes (below) have the same 8 working warps, so every call cuts and
//     adds the sums alike: the result is the same, bit for bit, from call to
//     call.  Nothing crosses CTAs (no cluster, no global scratch), except the
//     greedy-decoding epilogue's last step: per-CTA maxima in a caller
//     workspace, reduced by the last CTA to finish (an atomic count).
//   * Zero point and scale are applied per block AFTER the tensor core, not
//     per weight.  The MMA (mma.sync m16n8k16, fp32 accumulation) takes the
//     raw codes: (nibble | 0x6400) is the fp16 1024+q exactly for a low
//     nibble, 1024+16q for a high nibble (met by x/16, staged exact), so 8
//     weights cost one shift and four LOP3.  With one token, 7 of the MMA's 8
//     columns would be wasted; instead column j collects block j of the box:
//     the x fragment of the thread whose column is j holds x only for the k of
//     block j, zeros elsewhere.  After a box the accumulator holds, for every
//     (row, block), D = sum_k (1024 + q~) x~, started from -P with
//     P = 1024 sum_k x~; the block's dot product is then
//     sum_k (q - zp) x = D - zp Q, Q = sum_k x (both sums per block of x,
//     computed once per call), and y += scale * (D - zp Q).  Four correction
//     FMAs per thread per box replace two half2 operations per weight pair.
//     The 16 MMAs of a box run as four independent accumulator chains: on
//     the decoder's small projections each warp holds one to three boxes, so
//     the latency of a chain, not the issue rate, sets the kernel's time.
//   * Consecutive launches alternate between two resource shapes that cannot
//     share an SM with themselves but can with each other, so the block
//     scheduler never puts two CTAs of one launch on an SM (launch_res_t).
//     The second shape's extra warps only widen it.  (Giving them units too
//     was measured slower over the decode step, and would make the two
//     shapes cut the sums differently.)
// Every mbarrier wait is bounded in time; past the limit the kernel records
// the failure in the device status word, lets its copies in flight land and
// exits.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace mnb {

__device__ unsigned g_res_status = 0;

namespace {

// Index checks of the debug build (MNB_DEVICE_CHECKS, built as libmnb_debug.so):
// an index outside [0, bound) sets bit 4 of the status word and is replaced by
// 0, so the access stays inside its buffer; nothing traps.  The release build
// compiles them away.
__device__ __forceinline__ int checked(int idx, int bound) {
#ifdef MNB_DEVICE_CHECKS
    if (idx < 0 || idx >= bound) {
        atomicOr(&g_res_status, 16u);
        return 0;
    }
#else
    (void)bound;
#endif
    return idx;
}

constexpr int kWarps = 8;                   // warps that work; a launch may add idle ones (see below)
constexpr int kThreads = kWarps * 32;
constexpr int kStreamWarps = 20;            // working warps of a weight stream's CTA
constexpr int kStreamCtas = 1;              // ... and its CTAs per SM
constexpr int kMaxThreads = 16 * 32;
constexpr int kMaxXWords = 4;              // 16-byte words of x per thread: K <= 8192
constexpr int kMaxRegs = 96;                // register cap of the kernel (the launch shapes depend on it)
constexpr int kRows = 16;
constexpr int kBoxK = 256;                  // k per box: 8 blocks of 32 (4 of 64)
constexpr int kBoxBytes = kRows * 128;
constexpr int kParBytes = 320;              // 16 rows x 16 B of scales, then 16 rows x 4 B of zero points
constexpr int kChunk = 80;                  // staged bytes per 32-k chunk of x: 64, then 16 of padding
constexpr int kMaxDepth = 8;
constexpr int kSmemBudget = 110 * 1024;     // two CTAs (of consecutive kernels) per SM
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

struct ResParams {
    const __half *X;          // [K]
    const uint8_t *scales;    // fp16 [N][nb]
    const uint8_t *zp;        // [N][zpb] or null (zero point 8)
    __half *Y;                // [N]
    int N, K, nb, zpb;
    int ntiles, nbx, nchunks; // ceil(N / 16), K / 256, K / 32
    int tq, tr;               // tiles per CTA: tq, one more for CTAs below tr
    int depth;                // ring slots per warp
    // greedy decoding: ids[0] = the first n of max y[n] (over the fp16 values
    // stored), max_out[0] its value; per-CTA partials in a caller workspace,
    // reduced by the last CTA to finish (counter in the workspace's header)
    int argmax;
    // SwiGLU epilogue: weight rows in 16-row groups, 8 gate rows then the 8 up
    // rows of the same outputs; y[8 t + i] = silu(gate) * up, N / 2 outputs
    int swiglu;
    int32_t *ids;
    float *max_out;
    uint2 *ws_part;           // [gridDim.x] (value bits, index)
    unsigned *ws_count;
};

// silu(x) = x * sigmoid(x), in fp32.
__device__ __forceinline__ float silu(float x) { return x / (1.0f + __expf(-x)); }

// (value, index) pairs ordered by value, then by the SMALLER index: the greedy
// token is the first maximum.
__device__ __forceinline__ void keep_best(float v, int i, float &bv, int &bi) {
    if (v > bv || (v == bv && i < bi)) {
        bv = v;
        bi = i;
    }
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// One arrival on `bar` once all of this thread's earlier cp.async copies have
// landed (the barrier's expected count includes it).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Bounded wait on a warp-private mbarrier; after the first timeout it returns
// at once, so the warp runs to the end without waiting again.
__device__ __forceinline__ void slot_wait(uint32_t bar, uint32_t parity, bool &dead) {
    if (dead || mbar_try_wait(bar, parity))
        return;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(bar, parity))
            return;
        if ((i & 255) == 0 && globaltimer() - t0 > kWaitLimitNs) {
            dead = true;
            atomicOr(&g_res_status, 1u);
            return;
        }
    }
}

// A warp's request cursor: the next unit (tile, box) and, for this lane, the
// global address of its parameter bytes of that box (lanes 0-15: the scales of
// row n0 + lane; lanes 16-31: the zero points of row n0 + lane - 16) and
// whether that row exists.  Advancing by a box is a pointer increment; only a
// new tile recomputes the addresses.
struct IssueCursor {
    int tile, box;
    const uint8_t *src;
    bool row_ok;
};

template <bool BS64, bool ZP>
__device__ __forceinline__ void cursor_at_tile(const ResParams &p, IssueCursor &q, int tile, int box, int lane) {
    q.tile = tile;
    q.box = box;
    const int n = tile * kRows + (lane & 15);
    q.row_ok = n < p.N;
    if (lane < 16)
        q.src = p.scales + ((int64_t)n * p.nb + box * (BS64 ? 4 : 8)) * 2;
    else
        q.src = ZP ? p.zp + (int64_t)n * p.zpb + (BS64 ? (box >> 1) * 4 : box * 4) : nullptr;
}

template <bool BS64, bool ZP>
__device__ __forceinline__ void cursor_next(const ResParams &p, IssueCursor &q, int lane) {
    if (++q.box == p.nbx) {
        cursor_at_tile<BS64, ZP>(p, q, q.tile + 1, 0, lane);
        return;
    }
    if (lane < 16)
        q.src += BS64 ? 8 : 16;
    else if (ZP && (!BS64 || (q.box & 1) == 0))
        q.src += 4;   // block 64: one 4-byte load of zero points serves two boxes
}

// Requests the cursor's unit into a ring slot: the packed box by TMA (lane 0),
// the box's scales (lanes 0-15) and zero points (lanes 16-31) by cp.async.
// Rows past N get no parameters (their sums are never stored).  Every lane
// arrives on the slot's barrier once its copies have landed.
// A weight box by TMA, marked first to leave L2: each box is read once per
// call, while a row's scales and zero points come in 32-byte sectors that
// the row's next box reads again (the lm_head: 1.044x the algorithmic DRAM
// bytes without the hint).
__device__ __forceinline__ void tma_load_2d_evict_first(uint32_t dst, const void *map, uint32_t bar, int x, int y) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y), "l"(pol)
        : "memory");
}

template <bool BS64, bool ZP>
__device__ __forceinline__ void issue(const CUtensorMap *wmap, const ResParams &p, const IssueCursor &q,
                                      uint32_t box_dst, uint32_t par_dst, uint32_t full, int lane) {
    if (lane == 0) {
        mbar_expect_tx(full, kBoxBytes);
        tma_load_2d_evict_first(box_dst, wmap, full, checked(q.box, p.nbx) * 128, checked(q.tile, p.ntiles) * kRows);
    }
    if (q.row_ok) {
        if (lane < 16) {
            if (BS64) cp_async_8(par_dst + lane * 16, q.src); else cp_async_16(par_dst + lane * 16, q.src);
        } else if (ZP) {
            cp_async_4(par_dst + 256 + (lane - 16) * 4, q.src);
        }
    }
    cp_async_arrive(full);
}

// Scales of the box's columns 2c and 2c+1 (32-k chunks) of a row, from its
// slot's parameter area, as fp32.
template <bool BS64>
__device__ __forceinline__ float2 scale_pair(const unsigned char *par, int row, int c) {
    if (!BS64) {   // blocks 2c, 2c+1
        const uint32_t v = *reinterpret_cast<const uint32_t *>(par + row * 16 + c * 4);
        return __half22float2(u32_as_h2(v));
    }
    // block 64: columns 2c, 2c+1 are the two halves of block c of the box
    const float s = __half2float(__ushort_as_half(*reinterpret_cast<const unsigned short *>(par + row * 16 + c * 2)));
    return make_float2(s, s);
}

// Zero points of columns 2c, 2c+1 of a row, as fp32.
template <bool BS64, bool ZP>
__device__ __forceinline__ float2 zp_pair(const unsigned char *par, int row, int c, int box) {
    if (!ZP)
        return make_float2(8.f, 8.f);
    // a nibble z as fp32 without the conversion unit: (2^23 + z) - 2^23
    if (!BS64) {
        const uint32_t zb = par[256 + row * 4 + c];   // blocks 2c (low nibble) and 2c+1 (high)
        return make_float2(__uint_as_float(0x4B000000u | (zb & 15u)) - 8388608.f,
                           __uint_as_float(0x4B000000u | (zb >> 4)) - 8388608.f);
    }
    const uint32_t zb = par[256 + row * 4 + (box & 1) * 2 + (c >> 1)];
    const float z = __uint_as_float(0x4B000000u | ((c & 1) ? (zb >> 4) : (zb & 15u))) - 8388608.f;
    return make_float2(z, z);
}

template <bool BS64, bool ZP, int NW>
__global__ void __maxnreg__(kMaxRegs)
    gemv_resident_kernel(const __grid_constant__ CUtensorMap wmap, const ResParams p) {
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int D = p.depth;

    // shared memory (1024-aligned): boxes | params | x | zero chunk | (P, Q) |
    // partial sums | their tiles | barriers
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *bp = smem_raw + (base - smem_u32(smem_raw));
    unsigned char *pars = bp + NW * D * kBoxBytes;
    unsigned char *xs = pars + NW * D * kParBytes;
    unsigned char *zchunk = xs + p.nchunks * kChunk;
    float2 *pq = reinterpret_cast<float2 *>(zchunk + kChunk);
    float *part = reinterpret_cast<float *>(pq + p.nchunks);      // [warp][2 slots][16 rows]
    int *part_tile = reinterpret_cast<int *>(part + NW * 2 * kRows);
    uint2 *wbest = reinterpret_cast<uint2 *>(part_tile + NW * 2);   // greedy decoding: per warp
    const uint32_t bars = smem_u32(wbest + NW);
    const uint32_t my_box = base + (uint32_t)(warp * D * kBoxBytes);
    const unsigned char *my_box_ptr = bp + warp * D * kBoxBytes;
    const uint32_t my_par = smem_u32(pars) + (uint32_t)(warp * D * kParBytes);
    const unsigned char *my_par_ptr = pars + warp * D * kParBytes;
    const uint32_t my_bars = bars + (uint32_t)(warp * D * 8);
    // warps beyond NW only widen the launch (so that two CTAs of one
    // launch cannot share an SM): no units, no barriers, no slots; they take
    // part in the CTA barriers only
    const bool worker = warp < NW;

    // this CTA's tiles and this warp's run of (tile, box) units
    const int cta = blockIdx.x;
    const int Tc = p.tq + (cta < p.tr ? 1 : 0);
    const int t0 = cta * p.tq + (cta < p.tr ? cta : p.tr);
    const int U = Tc * p.nbx;
    const int u0 = (worker ? warp : NW) * U / NW, u1 = (worker ? warp + 1 : NW) * U / NW;

    if (worker && lane == 0) {
        for (int d = 0; d < D; d++)
            mbar_init(my_bars + 8 * d, 33);   // lane 0's expect_tx + one cp.async arrival per lane
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < NW * 2)
        part_tile[tid] = -1;
    __syncwarp();

    // ---- weights first: they do not depend on the previous kernel
    const int tl0 = u0 / p.nbx;          // this warp's first unit
    const int box0 = u0 - tl0 * p.nbx;
    int iu = u0, islot = 0;              // next unit to request, its slot
    IssueCursor ic;
    cursor_at_tile<BS64, ZP>(p, ic, t0 + tl0, box0, lane);
    auto request = [&]() {
        issue<BS64, ZP>(&wmap, p, ic, my_box + islot * kBoxBytes, my_par + islot * kParBytes, my_bars + 8 * islot, lane);
        cursor_next<BS64, ZP>(p, ic, lane);
        ++iu;
        if (++islot == D) islot = 0;
    };
    while (iu < u1 && iu - u0 < D)
        request();
    pdl_launch_dependents();
    pdl_wait();

    // ---- stage x: chunk j (k = 32j .. 32j+31) as four 16-byte words, word w =
    // (x0,x4) (x1,x5)/16 (x2,x6) (x3,x7)/16 of k = 32j + 8w ..; and per chunk
    // P = 1024 sum x~ and Q = sum x over the staged values x~ (x/16 counted
    // back as 16 x~), so the correction matches the MMA's operands exactly.
    // One 16-byte word per thread per pass (K / 8 is a multiple of 32, so every
    // lane of a warp takes part in each pass); the four words of a chunk sit in
    // four consecutive lanes, which add their sums by shuffles.
    {
        const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
        // every load first (up to four per thread), then the stores: one
        // trip to L2 on the critical path, whatever K
        uint4 vv[kMaxXWords];
#pragma unroll
        for (int r = 0; r < kMaxXWords; r++) {
            const int u = tid + r * (NW * 32);
            if (worker && u < p.nchunks * 4)
                vv[r] = ldg_v4(p.X + 8 * u);
        }
#pragma unroll
        for (int r = 0; r < kMaxXWords; r++) {
            const int u = tid + r * (NW * 32);
            if (!worker || u >= p.nchunks * 4)   // warp-uniform: K / 8 is a multiple of 32
                break;
            const int j = u >> 2, w = u & 3;
            const uint4 v = vv[r];
            uint4 o;
            o.x = __byte_perm(v.x, v.z, 0x5410);
            o.y = h2_as_u32(__hmul2(u32_as_h2(__byte_perm(v.x, v.z, 0x7632)), sixteenth));
            o.z = __byte_perm(v.y, v.w, 0x5410);
            o.w = h2_as_u32(__hmul2(u32_as_h2(__byte_perm(v.y, v.w, 0x7632)), sixteenth));
            *reinterpret_cast<uint4 *>(xs + j * kChunk + w * 16) = o;
            const float2 a = __half22float2(u32_as_h2(o.x)), b = __half22float2(u32_as_h2(o.y));
            const float2 e = __half22float2(u32_as_h2(o.z)), f = __half22float2(u32_as_h2(o.w));
            float lo = (a.x + a.y) + (e.x + e.y);   // the low-position x
            float hi = (b.x + b.y) + (f.x + f.y);   // the high-position x~
            lo += __shfl_xor_sync(0xffffffffu, lo, 1);
            hi += __shfl_xor_sync(0xffffffffu, hi, 1);
            lo += __shfl_xor_sync(0xffffffffu, lo, 2);
            hi += __shfl_xor_sync(0xffffffffu, hi, 2);
            if (w == 0)
                pq[j] = make_float2(1024.f * (lo + hi), lo + 16.f * hi);
        }
        if (tid < kChunk / 16)
            reinterpret_cast<uint4 *>(zchunk)[tid] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    // ---- this warp's units
    bool dead = false;
    int cslot = 0, cph = 0;
    float ya = 0.f, yb = 0.f;   // rows g and g+8 of the current tile segment
    bool seg_from0 = false;
    int nseg = 0;               // segments of this warp emitted so far
    float best_v = -INFINITY;   // greedy decoding: this thread's best stored logit
    int best_i = 0x7fffffff;
    const int hm = g - 2 * c;   // the half (0 or 1) in which this thread's column takes x, if any
    int tl = tl0, box = box0;   // the unit being consumed (CTA-local tile, box)
    for (int u = u0; u < u1; u++, box = (box + 1 == p.nbx) ? 0 : box + 1, tl += (box == 0) ? 1 : 0) {
        if (u == u0 || box == 0) {
            ya = yb = 0.f;
            seg_from0 = (box == 0);
        }
        slot_wait(my_bars + 8 * cslot, (uint32_t)cph, dead);
        dead = __any_sync(0xffffffffu, dead);   // one verdict per warp: it issues refills together
        const unsigned char *bx = my_box_ptr + checked(cslot, D) * kBoxBytes;
        const unsigned char *par = my_par_ptr + checked(cslot, D) * kParBytes;
        const float4 pqv = *reinterpret_cast<const float4 *>(pq + checked(box * 8 + 2 * c, p.nchunks - 1));   // P, Q of columns 2c, 2c+1
        // four independent MMA chains (half of the box x parity of the word),
        // the first started from -P: the 16 MMAs of a box form chains of four
        float acc4[4][4] = {{-pqv.x, -pqv.z, -pqv.x, -pqv.z}, {0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f},
                            {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int chunk = 2 * c + h;
            const uint4 va = *reinterpret_cast<const uint4 *>(bx + g * 128 + ((chunk ^ g) << 4));
            const uint4 vb = *reinterpret_cast<const uint4 *>(bx + (g + 8) * 128 + ((chunk ^ g) << 4));
            // x of chunk `chunk` goes to column `chunk` only: the thread whose
            // column that is (g == chunk) reads it, every other thread zeros
            const unsigned char *xa = (hm == h) ? xs + checked(box * 8 + chunk, p.nchunks) * kChunk : zchunk;
            const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
            const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xa + w * 16);
                const uint32_t a8 = wa[w] >> 8, b8 = wb[w] >> 8;
                const uint32_t a0 = lop3_and_or(wa[w], 0x000F000Fu, 0x64006400u);   // (e0, e4): 1024 + q
                const uint32_t a1 = lop3_and_or(wa[w], 0x00F000F0u, 0x64006400u);   // (e1, e5): 1024 + 16 q
                const uint32_t a2 = lop3_and_or(a8, 0x000F000Fu, 0x64006400u);      // (e2, e6)
                const uint32_t a3 = lop3_and_or(a8, 0x00F000F0u, 0x64006400u);      // (e3, e7)
                const uint32_t b0 = lop3_and_or(wb[w], 0x000F000Fu, 0x64006400u);
                const uint32_t b1 = lop3_and_or(wb[w], 0x00F000F0u, 0x64006400u);
                const uint32_t b2 = lop3_and_or(b8, 0x000F000Fu, 0x64006400u);
                const uint32_t b3 = lop3_and_or(b8, 0x00F000F0u, 0x64006400u);
                float *acc = acc4[2 * h + (w & 1)];
                mma16816(acc, a0, b0, a1, b1, xv.x, xv.y);
                mma16816(acc, a2, b2, a3, b3, xv.z, xv.w);
            }
        }
        // correction: columns 2c, 2c+1 of rows g and g+8
        {
            float acc[4];
#pragma unroll
            for (int e = 0; e < 4; e++) acc[e] = (acc4[0][e] + acc4[1][e]) + (acc4[2][e] + acc4[3][e]);
            const float2 sa = scale_pair<BS64>(par, g, c), sb = scale_pair<BS64>(par, g + 8, c);
            const float2 za = zp_pair<BS64, ZP>(par, g, c, box), zb = zp_pair<BS64, ZP>(par, g + 8, c, box);
            if (!dead) {
                ya = fmaf(sa.x, fmaf(-za.x, pqv.y, acc[0]), ya);
                ya = fmaf(sa.y, fmaf(-za.y, pqv.w, acc[1]), ya);
                yb = fmaf(sb.x, fmaf(-zb.x, pqv.y, acc[2]), yb);
                yb = fmaf(sb.y, fmaf(-zb.y, pqv.w, acc[3]), yb);
            }
        }
        __syncwarp();
        if (++cslot == D) { cslot = 0; cph ^= 1; }
        if (!dead && iu < u1) {
            fence_proxy_async_smem();   // this warp's reads of the slot precede the TMA that refills it
            request();
        }
        // ---- end of a tile segment
        if (box == p.nbx - 1 || u + 1 == u1) {
            ya += __shfl_xor_sync(0xffffffffu, ya, 1);
            ya += __shfl_xor_sync(0xffffffffu, ya, 2);
            yb += __shfl_xor_sync(0xffffffffu, yb, 1);
            yb += __shfl_xor_sync(0xffffffffu, yb, 2);
            const int tile = t0 + tl;
            if (seg_from0 && box == p.nbx - 1) {
                if (c == 0 && !dead && p.swiglu) {   // row g is a gate, row g + 8 its up
                    if (tile * kRows + g < p.N)
                        p.Y[tile * 8 + g] = __float2half_rn(silu(ya) * yb);
                } else if (c == 0 && !dead) {
                    const int n = tile * kRows + g;
                    const __half ha = __float2half_rn(ya), hb = __float2half_rn(yb);
                    if (n < p.N) {
                        p.Y[n] = ha;
                        keep_best(__half2float(ha), n, best_v, best_i);
                    }
                    if (n + 8 < p.N) {
                        p.Y[n + 8] = hb;
                        keep_best(__half2float(hb), n + 8, best_v, best_i);
                    }
                }
            } else {
                // a partial: the first segment of the run in slot 0, the last in slot 1
                const int s = checked(warp * 2 + ((nseg == 0) ? 0 : 1), NW * 2);
                if (c == 0) {
                    part[s * kRows + g] = ya;
                    part[s * kRows + g + 8] = yb;
                }
                if (lane == 0)
                    part_tile[s] = tile;
            }
            ++nseg;
        }
    }
    __syncthreads();

    // ---- tiles cut between warps: the first warp slot holding a tile adds
    // every slot holding it, in warp order, and stores the rows.  The slots'
    // tiles are read once into registers, so the scan and the sum are not
    // chains of dependent shared-memory reads.
    {
        const int sl = tid >> 4, row = tid & 15;   // 2 NW slots x 16 rows = the working warps' threads
        int tiles[NW * 2];
#pragma unroll
        for (int q = 0; q < NW * 2; q += 4) {
            const int4 t4 = *reinterpret_cast<const int4 *>(part_tile + q);
            tiles[q] = t4.x; tiles[q + 1] = t4.y; tiles[q + 2] = t4.z; tiles[q + 3] = t4.w;
        }
        int tile = -1;
#pragma unroll
        for (int q = 0; q < NW * 2; q++)
            if (q == sl) tile = tiles[q];
        bool leader = worker && tile >= 0;
#pragma unroll
        for (int q = 0; q < NW * 2; q++)
            if (q < sl && tiles[q] == tile) leader = false;
        if (leader && p.swiglu) {   // rows < 8: the gates; row + 8: their ups
            if (row < 8) {
                float gv = 0.f, uv = 0.f;
#pragma unroll
                for (int q = 0; q < NW * 2; q++)
                    if (q >= sl && tiles[q] == tile) {
                        gv += part[q * kRows + row];
                        uv += part[q * kRows + row + 8];
                    }
                if (tile * kRows + row < p.N && !dead)
                    p.Y[tile * 8 + row] = __float2half_rn(silu(gv) * uv);
            }
        } else if (leader) {
            float v = 0.f;
#pragma unroll
            for (int q = 0; q < NW * 2; q++)
                if (q >= sl && tiles[q] == tile)
                    v += part[q * kRows + row];
            const int n = tile * kRows + row;
            if (n < p.N && !dead) {
                const __half h = __float2half_rn(v);
                p.Y[n] = h;
                keep_best(__half2float(h), n, best_v, best_i);
            }
        }
    }

    // ---- greedy decoding: the CTA's best into the workspace; the last CTA
    // to finish reduces every CTA's and resets the counter for the next call
    if (p.argmax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
            const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
            keep_best(ov, oi, best_v, best_i);
        }
        if (worker && lane == 0)
            wbest[warp] = make_uint2(__float_as_uint(best_v), (unsigned)best_i);
        __syncthreads();
        __shared__ int s_last;
        if (tid == 0) {
            float v = -INFINITY;
            int i = 0x7fffffff;
            for (int w = 0; w < NW; w++)
                keep_best(__uint_as_float(wbest[w].x), (int)wbest[w].y, v, i);
            p.ws_part[blockIdx.x] = make_uint2(__float_as_uint(v), (unsigned)i);
            __threadfence();
            s_last = (atomicAdd(p.ws_count, 1u) == gridDim.x - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            float v = -INFINITY;
            int i = 0x7fffffff;
            for (int b = tid; worker && b < (int)gridDim.x; b += (NW * 32)) {
                const uint2 e = __ldcg(p.ws_part + b);
                keep_best(__uint_as_float(e.x), (int)e.y, v, i);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, v, o);
                const int oi = __shfl_xor_sync(0xffffffffu, i, o);
                keep_best(ov, oi, v, i);
            }
            if (worker && lane == 0)
                wbest[warp] = make_uint2(__float_as_uint(v), (unsigned)i);
            __syncthreads();
            if (tid == 0) {
                for (int w = 1; w < NW; w++)
                    keep_best(__uint_as_float(wbest[w].x), (int)wbest[w].y, v, i);
                p.ids[0] = i;
                if (p.max_out)
                    p.max_out[0] = v;
                *p.ws_count = 0u;   // ready for the next call
            }
        }
    }

    // after a timeout: let the copies still in flight (at most one ring's
    // worth) land before the CTA's shared memory is released
    if (dead && lane == 0) {
        const int issued = iu - u0;
        for (int q = (issued > D ? issued - D : 0); q < issued; q++) {
            const uint32_t bar = my_bars + 8 * (q % D);
            const unsigned long long tw = globaltimer();
            while (!mbar_try_wait(bar, (uint32_t)((q / D) & 1)) && globaltimer() - tw < kWaitLimitNs) {
            }
        }
    }
}

size_t res_smem_bytes(int nw, int depth, int nchunks) {
    return 1024 + (size_t)nw * depth * (kBoxBytes + kParBytes + 8) + (size_t)nchunks * (kChunk + 8) + kChunk +
           (size_t)nw * 2 * (kRows * 4 + 4) + (size_t)nw * 8;
}

// The deepest ring (up to the most units a warp owns) for nw working warps
// within `budget` bytes of shared memory; 0 when none fits.
int res_depth(int nw, int Umax, int nchunks, size_t budget) {
    const int per_warp = (Umax + nw - 1) / nw;
    int depth = per_warp < kMaxDepth ? (per_warp < 2 ? 2 : per_warp) : kMaxDepth;
    while (depth > 2 && res_smem_bytes(nw, depth, nchunks) > budget)
        --depth;
    return res_smem_bytes(nw, depth, nchunks) <= budget ? depth : 0;
}

// Launch shapes.  The CTAs of kernel i+1 are placed while kernel i runs;
// where an SM has both halves free (kernel i had no CTA there, or its CTA has
// left) the block scheduler may put TWO CTAs of one launch on it, which then
// share the SM and double its part of the critical path.  Consecutive
// launches therefore alternate between two shapes that cannot pair with
// themselves but pair with each other: shape A asks for just over half of
// the SM's shared memory, shape B for just over half of the registers of
// each SM sub-partition (idle warps widen it; hence the kernel's register
// cap).  One A and one B fit on an SM; two of either do not.  A
// weight stream (the lm_head) takes one shape: a CTA with the whole SM, 20
// working warps (five per sub-partition, the most this kernel's registers
// allow).  Its time is set by how fast each warp gets through its boxes, so
// more warps per SM stream faster.
struct LaunchShape {
    int threads;
    size_t smem;
};

template <bool BS64, bool ZP, int NW>
int launch_res_t(const CUtensorMap &map, ResParams p, int grid, int depth, bool stream_mode, unsigned flags,
                 cudaStream_t s) {
    auto fn = gemv_resident_kernel<BS64, ZP, NW>;
    p.depth = depth;
    const size_t smem = res_smem_bytes(NW, depth, p.nchunks);
    static int regs[kMaxDevices] = {}, smem_sm[kMaxDevices] = {}, reserved[kMaxDevices] = {}, rf[kMaxDevices] = {};
    static std::atomic<unsigned> parity[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        dev = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (regs[dev] == 0) {
            cudaFuncAttributes a;
            cudaError_t e = cudaFuncGetAttributes(&a, fn);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(&smem_sm[dev], cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(&reserved[dev], cudaDevAttrReservedSharedMemoryPerBlock, dev);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(&rf[dev], cudaDevAttrMaxRegistersPerMultiprocessor, dev);
            if (e == cudaSuccess)   // both halves of an SM's shared memory to this kernel's shapes
                e = cudaFuncSetAttribute(reinterpret_cast<const void *>(fn),
                                         cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            if (e != cudaSuccess)
                return fail(MNB_ERR_CUDA, "mnb_gemv: kernel attributes: %s", cudaGetErrorString(e));
            regs[dev] = (a.numRegs + 7) & ~7;
        }
    }
    LaunchShape shape{NW * 32, smem};
    if (!stream_mode) {
        // registers are allocated per SM sub-partition (four per SM; a CTA's
        // warps go round-robin over them): cap = warps of this kernel one
        // sub-partition holds; A has kWarps / 4 per sub-partition, B just over
        // half of the cap, so A + B fits and B + B does not
        const int R = regs[dev];
        const int cap = (rf[dev] / 4) / (32 * R);
        const int a = kWarps / 4, b = cap / 2 + 1;
        const size_t smemA = (size_t)(smem_sm[dev] - 2 * reserved[dev]) / 2 + 1024;   // A: more than half
        const bool ok = a + b <= cap && 4 * b * 32 <= kMaxThreads &&
                        smemA + smem + 2 * (size_t)reserved[dev] <= (size_t)smem_sm[dev] && smem <= smemA;
        const int wB = 4 * b;
        if (ok) {
            if (parity[dev].fetch_add(1u, std::memory_order_relaxed) & 1u)
                shape.threads = 32 * wB;
            else
                shape.smem = smemA;
        }
    }
    static int configured[kMaxDevices] = {};
    {
        cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(fn), (int)shape.smem, configured);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemv: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)shape.threads, 1, 1);
    cfg.dynamicSmemBytes = shape.smem;
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, map, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

}  // namespace

int launch_gemv_resident(const void *X, const uint8_t *packed, const void *scales, const uint8_t *zp, void *Y, int N,
                         int K, int bs, unsigned flags, cudaStream_t s, int32_t *ids, float *max_out,
                         void *workspace, int swiglu) {
    const bool bs64 = (bs == 64), has_zp = (zp != nullptr);
    if (K % kBoxK != 0 || K > kMaxXWords * kThreads * 8 || (bs64 && has_zp && K % 512 != 0) ||
        !aligned(scales, bs64 ? 8 : 16) ||
        (has_zp && !aligned(zp, 4)))
        return 1;   // not a shape this kernel serves
    ResParams p;
    p.X = static_cast<const __half *>(X);
    p.scales = static_cast<const uint8_t *>(scales);
    p.zp = zp;
    p.Y = static_cast<__half *>(Y);
    p.N = N;
    p.K = K;
    p.nb = K / bs;
    p.zpb = (p.nb + 1) / 2;
    p.ntiles = (N + kRows - 1) / kRows;
    p.nbx = K / kBoxK;
    p.nchunks = K / 32;
    // one CTA per SM (the next kernel's CTAs take the other half); a weight
    // stream of more than 16 tiles per SM (the lm_head) takes both halves, as
    // 8 warps leave the SM with too few to hide their latency
    const int sms = device_sm_count();
    const bool stream_mode = p.ntiles > 16 * sms;
    const int grid = stream_mode ? kStreamCtas * sms : (p.ntiles < sms ? p.ntiles : sms);
    p.tq = p.ntiles / grid;
    p.tr = p.ntiles % grid;
    const int Umax = (p.tq + (p.tr ? 1 : 0)) * p.nbx;   // the most units of any CTA
    const int depth = res_depth(kWarps, Umax, p.nchunks, (size_t)kSmemBudget);
    const int depth_s = stream_mode ? res_depth(kStreamWarps, Umax, p.nchunks, (size_t)kSmemBudget * 2 / kStreamCtas) : 0;
    if (!depth)
        return 1;
    p.argmax = ids ? 1 : 0;
    p.swiglu = swiglu;
    p.ids = ids;
    p.max_out = max_out;
    p.ws_count = static_cast<unsigned *>(workspace);
    p.ws_part = workspace ? reinterpret_cast<uint2 *>(static_cast<unsigned char *>(workspace) + 256) : nullptr;

    EncodeTiledFn encode = tensor_map_encoder();
    if (!encode)
        return fail(MNB_ERR_CUDA, "mnb_gemv: cuTensorMapEncodeTiled unavailable");
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
    if (depth_s) {   // a weight stream: one shape, the wider CTAs
        if (bs64) {
            if (has_zp) return launch_res_t<true, true, kStreamWarps>(map, p, grid, depth_s, true, flags, s);
            return launch_res_t<true, false, kStreamWarps>(map, p, grid, depth_s, true, flags, s);
        }
        if (has_zp) return launch_res_t<false, true, kStreamWarps>(map, p, grid, depth_s, true, flags, s);
        return launch_res_t<false, false, kStreamWarps>(map, p, grid, depth_s, true, flags, s);
    }
    if (bs64) {
        if (has_zp) return launch_res_t<true, true, kWarps>(map, p, grid, depth, stream_mode, flags, s);
        return launch_res_t<true, false, kWarps>(map, p, grid, depth, stream_mode, flags, s);
    }
    if (has_zp) return launch_res_t<false, true, kWarps>(map, p, grid, depth, stream_mode, flags, s);
    return launch_res_t<false, false, kWarps>(map, p, grid, depth, stream_mode, flags, s);
}

int read_res_status(unsigned *out, int clear) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_res_status, sizeof(unsigned));
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_res_status, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_device_status: %s", cudaGetErrorString(e));
    *out |= v;   // bit 0, as the other decode kernels; bit 4: an index check of the debug build
    return MNB_OK;
}

}  // namespace mnb
