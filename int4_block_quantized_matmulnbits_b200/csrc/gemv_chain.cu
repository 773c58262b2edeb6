// gemv_chain.cu -- the decode step's MatMulNBits GEMVs as ONE persistent launch.
//
// Per generated token the decoders of "Qwen3-ASR-0.6B -- ONNX for the browser"
// and "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)" run 28 layers x 7 projections
// plus the lm_head ("Graph contracts": decoder_step).  Issued as one kernel
// each, that is a chain of ~200 dependent launches whose small members move
// 1-3 MB of weights -- well under a microsecond of HBM time -- but each pays a
// launch's fixed cost (drain, release of the next grid, its X staging).  Here
// one CTA per SM walks the whole list of GEMVs (the "tasks"):
//   * Each compute warp (15 per CTA; 11 or 7 when X needs the shared memory)
//     owns a ring of `depth` slots.  A slot holds one 16-row x 256-k weight
//     box (TMA, 128-byte swizzle) plus that box's scales and zero points
//     (cp.async, completing on the same mbarrier).  Each warp refills its ring
//     from its own future work, across task boundaries: weights never depend
//     on earlier tasks, so the weights of the next tasks are already in shared
//     memory while this one waits for its X.  Requests for later tasks are
//     issued after the current task is signalled, off its critical path.  The
//     tensor maps live in the plan in global memory, written before launch.
//   * Task j may read X only once tasks 0..j-1 are complete (when its `wait`
//     is set).  Completion is a per-task counter in global memory: once its
//     compute warps have stored their part of Y, a CTA's control warp (which
//     issues no copies, so its release waits for nothing else) adds one with
//     release semantics, and polls the counter of task j-1 with acquire loads.  The CTA that completes the last task returns every
//     counter to zero.
//   * Work split of a task: CTA b owns a contiguous run of 16-row tiles.  With
//     at least as many tiles as warps each warp takes whole tiles (full K, Y
//     stored from registers); with fewer, the CTA's (tile, box) units are cut
//     into one contiguous run per warp, partial sums meet in shared memory and
//     the last warp to finish a tile stores it.
//   * Dequantisation and the mma.sync m16n8k16 inner product are those of the
//     single-GEMV decode kernel: fp16_rn((q - zp) * scale) per weight, exact,
//     fp32 accumulation.
// Every wait is bounded (globaltimer).  Past the limit a CTA records the
// failure in a device status word and in the workspace's abort word, which the
// other CTAs poll; all CTAs then leave the task loop together, drain their
// copies and exit.  The counters are then left as they were: the caller zeroes
// the workspace before the next call, and a call that finds the abort word set
// runs no task (status bit) rather than trust stale counters.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "mnb_tune.h"

namespace mnb {

__device__ unsigned g_chain_status = 0;

namespace {

constexpr int kMaxWarps = 15;              // compute warps per CTA: 15, fewer when X is large
constexpr int kMaxThreads = (kMaxWarps + 1) * 32;   // and one control warp
constexpr int kRows = 16;
constexpr int kBoxK = 256;
constexpr int kBoxBytes = kRows * 128;
constexpr int kParBytes = 320;             // 16 rows x 16 B of scales, then 16 rows x 4 B of zero points
constexpr int kMaxSplitTiles = kMaxWarps - 1;   // a CTA with fewer tiles than warps splits K
constexpr int kMP = 8;                     // token columns of one m16n8k16 (M <= 8)
constexpr int kMaxDepth = 4;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr uint32_t kPlanMagic = 0x434E4D42u;   // "BMNC"
constexpr uint32_t kPlanVersion = 1;

// One GEMV of the chain, as the kernel reads it from the device copy of the plan.
struct alignas(64) ChainTask {
    CUtensorMap wmap;          // packed [N][K/2] bytes; box 128 B x 16 rows, 128-byte swizzle
    const __half *X;           // [M][K]
    const uint8_t *scales;     // fp16 [N][nb]
    const uint8_t *zp;         // [N][zpb] or null (zero point 8)
    __half *Y;                 // [M][N]
    int N, K, nb, zpb;
    int ntiles, nbx;           // N / 16, K / 256
    int tq, tr;                // tiles per CTA: tq, one more for CTAs below tr
    int wait;                  // read X only after every earlier task is complete
    int pad[7];
};
static_assert(sizeof(ChainTask) == 256, "plan layout");

// The plan's first 64 bytes: what the host needs to launch it.
struct alignas(64) ChainHeader {
    uint32_t magic, version;
    int ntasks, M, bs, has_zp, grid, depth, xs_stride, smem, device, nw;
    int pad[4];
};
static_assert(sizeof(ChainHeader) == 64, "plan layout");

// The fields of a task the kernel reads on its hot path, copied once per CTA
// into shared memory (with ~200 KB of shared memory per SM the L1 left for
// the plan is small, and every global read of it is an L2 round trip).
struct TaskInfo {
    const __half *X;
    __half *Y;
    const uint8_t *scales;
    const uint8_t *zp;
    int N, K, nb, zpb;
    int tq, tr, nbx, wait;
};
static_assert(sizeof(TaskInfo) == 64, "task table layout");

struct ChainParams {
    const ChainTask *tasks;
    unsigned *cnt;       // [ntasks] completion counters, then the abort word
    int ntasks, M, depth, xs_stride, nw;   // nw: compute warps per CTA
    // fault injection for tests of the timeout path (mnb_test_chain_withhold):
    // no CTA counts task `withhold` complete (-1: none), and a wait for a
    // task's inputs gives up after task_wait_ns
    int withhold;
    unsigned long long task_wait_ns;
};

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
__device__ __forceinline__ void red_release_gpu(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}



// Bounded wait on an mbarrier; after the first timeout it returns at once.
__device__ __forceinline__ void slot_wait(uint32_t bar, uint32_t parity, bool &dead) {
    if (dead || mbar_try_wait(bar, parity))
        return;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(bar, parity))
            return;
        if ((i & 255) == 0 && globaltimer() - t0 > kWaitLimitNs) {
            dead = true;
            atomicOr(&g_chain_status, 1u);
            return;
        }
    }
}

// The run of units one warp owns in a task.  Units are (tile, box) pairs in
// tile-major order over the CTA's contiguous run of tiles.
__device__ __forceinline__ void run_of(const TaskInfo *t, int nw, int cta, int w, int &u0, int &u1, int &t0) {
    const int tq = t->tq, tr = t->tr, nbx = t->nbx;
    const int Tc = tq + (cta < tr ? 1 : 0);
    t0 = cta * tq + (cta < tr ? cta : tr);
    if (Tc >= nw) {   // whole tiles per warp
        u0 = (w * Tc / nw) * nbx;
        u1 = ((w + 1) * Tc / nw) * nbx;
    } else {
        const int U = Tc * nbx;
        u0 = w * U / nw;
        u1 = (w + 1) * U / nw;
    }
}

// Requests one unit into a ring slot: the weight box by TMA (lane 0), the
// box's scales (lanes 0-15) and zero points (lanes 16-31) by cp.async.  Every
// lane arrives on the slot's `full` barrier when its copies land.
template <bool BS64, bool ZP>
__device__ __forceinline__ void issue(const CUtensorMap *wmap, const TaskInfo *t, int tile, int box, uint32_t box_dst,
                                      uint32_t par_dst, uint32_t full, int lane) {
    const int n0 = tile * kRows;
    if (lane == 0) {
        mbar_expect_tx(full, kBoxBytes);
        tma_load_2d(box_dst, wmap, full, box * 128, n0);
    }
    if (lane < 16) {
        const uint8_t *src = t->scales + ((int64_t)(n0 + lane) * t->nb + box * (BS64 ? 4 : 8)) * 2;
        if (BS64) cp_async_8(par_dst + lane * 16, src); else cp_async_16(par_dst + lane * 16, src);
    } else if (ZP) {
        const int row = lane - 16;
        const uint8_t *src = t->zp + (int64_t)(n0 + row) * t->zpb + (BS64 ? (box >> 1) * 4 : box * 4);
        cp_async_4(par_dst + 256 + row * 4, src);
    }
    cp_async_arrive(full);
}


// A warp's position in its own sequence of units across the tasks: task, unit
// within the warp's run of that task (u == u1 once the run is exhausted), and
// the unit's tile and box.
struct Cursor {
    int task, u, u1, tile, box, nbx;
};

// Moves c to the first unit of the first task >= from in which warp w has work
// (task = ntasks when there is none).
__device__ __forceinline__ void cursor_seek(const TaskInfo *ti, int ntasks, int nw, int cta, int w, Cursor &c,
                                            int from) {
    for (int j = from; j < ntasks; j++) {
        int u0, u1, t0;
        run_of(ti + j, nw, cta, w, u0, u1, t0);
        if (u1 > u0) {
            c.task = j;
            c.u = u0;
            c.u1 = u1;
            c.nbx = ti[j].nbx;
            c.tile = t0 + u0 / c.nbx;
            c.box = u0 - (c.tile - t0) * c.nbx;
            return;
        }
    }
    c.task = ntasks;
    c.u = c.u1 = 0;
}

__device__ __forceinline__ void cursor_next(Cursor &c) {
    ++c.u;
    if (++c.box == c.nbx) {
        c.box = 0;
        ++c.tile;
    }
}

template <bool BS64, bool ZP>
__global__ void __launch_bounds__(kMaxThreads, 1) gemv_chain_kernel(const ChainParams p) {
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int cta = blockIdx.x;
    const unsigned grid = gridDim.x;
    const int D = p.depth, M = p.M, NW = p.nw, NT = (NW + 1) * 32;   // NW compute warps, then the control warp
    const bool control = (warp == NW);
    const int ctl = NW * 32;   // the thread that waits for and signals task completion

    // shared memory: boxes (1024-aligned) | box params | task table | X | zero
    // row | partial sums | their counters | flags | barriers
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *bp = smem_raw + (base - smem_u32(smem_raw));
    unsigned char *pars = bp + NW * D * kBoxBytes;
    TaskInfo *ti = reinterpret_cast<TaskInfo *>(pars + NW * D * kParBytes);
    unsigned char *xs = reinterpret_cast<unsigned char *>(ti + p.ntasks);
    unsigned char *zrow = xs + M * p.xs_stride;      // activations of tokens >= M
    float *red = reinterpret_cast<float *>(zrow + 512);
    int *red_cnt = reinterpret_cast<int *>(red + kMaxSplitTiles * kRows * kMP);   // warps done with a split tile
    int *flags = red_cnt + 16;   // [0]: abort
    const uint32_t bars = smem_u32(flags + 16);
    const uint32_t my_box = base + (uint32_t)(warp * D * kBoxBytes);
    const unsigned char *my_box_ptr = bp + warp * D * kBoxBytes;
    const uint32_t my_par = smem_u32(pars) + (uint32_t)(warp * D * kParBytes);
    const unsigned char *my_par_ptr = pars + warp * D * kParBytes;
    const uint32_t my_bars = bars + (uint32_t)(warp * D * 8);

    if (!control && lane == 0) {
        for (int d = 0; d < D; d++)
            mbar_init(my_bars + 8 * d, 33);   // lane 0's expect_tx + one cp.async arrival per lane
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the task table (the plan is in place before the previous kernel starts)
    for (int j = tid; j < p.ntasks; j += NT) {
        const ChainTask *t = p.tasks + j;
        TaskInfo v;
        v.X = t->X;
        v.Y = t->Y;
        v.scales = t->scales;
        v.zp = t->zp;
        v.N = t->N;
        v.K = t->K;
        v.nb = t->nb;
        v.zpb = t->zpb;
        v.tq = t->tq;
        v.tr = t->tr;
        v.nbx = t->nbx;
        v.wait = t->wait;
        ti[j] = v;
    }
    for (int i = tid; i < 128; i += NT)
        reinterpret_cast<uint32_t *>(zrow)[i] = 0u;
    for (int i = tid; i < kMaxSplitTiles * kRows * kMP; i += NT)
        red[i] = 0.f;
    if (tid < 32)
        red_cnt[tid] = 0;   // red_cnt[16] and flags[16]
    __syncthreads();

    // ---- the ring: issued and consumed counts, the next slot to fill, the
    // next unit to request.  Weights do not depend on earlier kernels or tasks:
    // the first units go out before waiting for the previous kernel.
    Cursor ic;
    int icount = 0, ccount = 0, islot = 0, cslot = 0, cph = 0;
    bool dead = false;
    auto refill = [&](int limit_task) {
        // request units until the ring is full, stopping before task limit_task
        while (icount - ccount < D) {
            if (ic.u == ic.u1)
                cursor_seek(ti, p.ntasks, NW, cta, warp, ic, ic.task + 1);
            if (ic.task >= limit_task)
                break;
            issue<BS64, ZP>(&p.tasks[ic.task].wmap, ti + ic.task, ic.tile, ic.box, my_box + islot * kBoxBytes,
                            my_par + islot * kParBytes, my_bars + 8 * islot, lane);
            ++icount;
            if (++islot == D) islot = 0;
            cursor_next(ic);
        }
    };
    if (!control) {
        ic.task = -1;
        ic.u = ic.u1 = 0;
        refill(p.ntasks);
    }
    pdl_wait();
    const half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
    // an abort word left set by a call that failed: the counters may be stale,
    // so run nothing (the caller zero-fills the workspace again)
    if (tid == ctl && ld_acquire_gpu(p.cnt + p.ntasks) != 0u) {
        flags[0] = 1;
        atomicOr(&g_chain_status, 4u);
    }
    __syncthreads();
    const int ntasks_run = flags[0] ? 0 : p.ntasks;

    for (int j = 0; j < ntasks_run; j++) {
        const TaskInfo *t = ti + j;
        const int nbx = t->nbx, N = t->N;
        __half *Y = t->Y;
        int u0 = 0, u1 = 0, t0 = 0;
        if (!control)
            run_of(t, NW, cta, warp, u0, u1, t0);
        if (j > 0 && t->wait) {
            // ---- X of task j is the output of earlier tasks: wait for all CTAs
            if (tid == ctl) {
                const unsigned *cp = p.cnt + (j - 1);
                if (ld_acquire_gpu(cp) < grid) {
                    const unsigned long long tw = globaltimer();
                    for (uint32_t i = 1;; i++) {
                        if (ld_acquire_gpu(cp) >= grid)
                            break;
                        if ((i & 63) == 0 &&
                            (ld_acquire_gpu(p.cnt + p.ntasks) != 0u || globaltimer() - tw > p.task_wait_ns)) {
                            flags[0] = 1;
                            atomicOr(&g_chain_status, 2u);
                            atomicExch(p.cnt + p.ntasks, 1u);
                            break;
                        }
                    }
                }
            }
            __syncthreads();
            if (flags[0])
                break;
        }

        // ---- stage X[0:M, 0:K) of task j.  Box qb, unit (h, w, cc) holds
        // k = qb*256 + (2cc+h)*32 + 8w .. +7 as (x0,x4) (x1,x5)/16 (x2,x6) (x3,x7)/16
        {
            const __half *X = t->X;
            const int K = t->K, per_tok = nbx * 8;
            for (int u = tid; u < M * per_tok; u += NT) {
                const int m = u / per_tok;
                const int r = u - m * per_tok;
                const int qb = r >> 3, chunk = r & 7;
                const int h = chunk & 1, cc = chunk >> 1;
                const int k = qb * kBoxK + chunk * 32;
                uint4 vv[4];
#pragma unroll
                for (int w = 0; w < 4; w++)
                    vv[w] = ldg_v4(X + (int64_t)m * K + k + 8 * w);
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
        }
        __syncthreads();

        // ---- this warp's units of task j
        int tile = t0 + (u1 > u0 ? u0 / nbx : 0);
        int box = (u1 > u0) ? u0 - (tile - t0) * nbx : 0;
        float acc[2][2][4];   // [chunk 2c + h][word parity]: four independent MMA chains
#pragma unroll
        for (int e = 0; e < 16; e++) acc[e >> 3][(e >> 2) & 1][e & 3] = 0.f;
        bool from0 = (box == 0);   // the current tile was started at box 0
        for (int u = u0; u < u1; u++) {
            slot_wait(my_bars + 8 * cslot, (uint32_t)cph, dead);
            if (!dead) {
                const unsigned char *bx = my_box_ptr + cslot * kBoxBytes;
                const unsigned char *par = my_par_ptr + cslot * kParBytes;
                uint32_t sA[2], sB[2], zA[2], zB[2];
                if (!BS64) {   // chunks 2c, 2c+1 = blocks 2c, 2c+1 of the box
                    const uint32_t pa = *reinterpret_cast<const uint32_t *>(par + g * 16 + c * 4);
                    const uint32_t pb = *reinterpret_cast<const uint32_t *>(par + (g + 8) * 16 + c * 4);
                    sA[0] = pa & 0xFFFFu; sA[1] = pa >> 16;
                    sB[0] = pb & 0xFFFFu; sB[1] = pb >> 16;
                    if (ZP) {
                        const uint32_t za = par[256 + g * 4 + c], zb = par[256 + (g + 8) * 4 + c];
                        zA[0] = za & 15u; zA[1] = za >> 4;
                        zB[0] = zb & 15u; zB[1] = zb >> 4;
                    } else {
                        zA[0] = zA[1] = zB[0] = zB[1] = 8u;
                    }
                } else {       // both chunks in block c of the box
                    sA[0] = sA[1] = *reinterpret_cast<const unsigned short *>(par + g * 16 + c * 2);
                    sB[0] = sB[1] = *reinterpret_cast<const unsigned short *>(par + (g + 8) * 16 + c * 2);
                    if (ZP) {
                        const int zo = 256 + (box & 1) * 2 + (c >> 1);
                        const uint32_t za = par[zo + g * 4], zb = par[zo + (g + 8) * 4];
                        zA[0] = zA[1] = (c & 1) ? (za >> 4) : (za & 15u);
                        zB[0] = zB[1] = (c & 1) ? (zb >> 4) : (zb & 15u);
                    } else {
                        zA[0] = zA[1] = zB[0] = zB[1] = 8u;
                    }
                }
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    const int chunk = 2 * c + h;
                    const uint4 va = *reinterpret_cast<const uint4 *>(bx + g * 128 + ((chunk ^ g) << 4));
                    const uint4 vb = *reinterpret_cast<const uint4 *>(bx + (g + 8) * 128 + ((chunk ^ g) << 4));
                    const uint32_t sa = sA[h] | (sA[h] << 16), sb = sB[h] | (sB[h] << 16);
                    const uint32_t Za = 0x64006400u | (zA[h] * 0x00010001u), Zb = 0x64006400u | (zB[h] * 0x00010001u);
                    const uint32_t Zha = 0x64006400u | (zA[h] * 0x00100010u), Zhb = 0x64006400u | (zB[h] * 0x00100010u);
                    const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
                    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
                    const unsigned char *xa = (g < M) ? xs + g * p.xs_stride + box * 512 + h * 256 + c * 16
                                                      : zrow + h * 256 + c * 16;
#pragma unroll
                    for (int w = 0; w < 4; w++) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(xa + w * 64);
                        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                        dq_word(wa[w], sa, Za, Zha, a0, a1, a2, a3);
                        dq_word(wb[w], sb, Zb, Zhb, b0, b1, b2, b3);
                        mma16816(acc[h][w & 1], a0, b0, a1, b1, xv.x, xv.y);
                        mma16816(acc[h][w & 1], a2, b2, a3, b3, xv.z, xv.w);
                    }
                }
            }
            ++ccount;
            if (++cslot == D) { cslot = 0; cph ^= 1; }
            __syncwarp();
            // a unit of this same task still waiting for a slot goes out now;
            // units of later tasks wait until this task is signalled
            if (!dead && ic.task == j && ic.u < ic.u1)
                refill(j + 1);
            const bool tile_end = (box == nbx - 1);
            if (tile_end || u + 1 == u1) {
                // ---- the warp is done with this tile: whole tiles go to Y;
                // split tiles meet in the shared partial sums, and the last of
                // their warps stores them
                const bool direct = from0 && tile_end;
                const int l = tile - t0;
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; e++)
                    v[e] = (acc[0][0][e] + acc[0][1][e]) + (acc[1][0][e] + acc[1][1][e]);
                if (direct) {
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int m = 2 * c + (e & 1);
                        if (m < M && !dead)
                            Y[(int64_t)m * N + tile * kRows + g + 8 * (e >> 1)] = __float2half_rn(v[e]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int m = 2 * c + (e & 1);
                        if (m < M)
                            atomicAdd(&red[(l * kRows + g + 8 * (e >> 1)) * kMP + m], v[e]);
                    }
                    // warps whose run meets tile l: one lane per warp checks
                    int a0 = 0, a1 = 0, at0 = 0;
                    if (lane < NW)
                        run_of(t, NW, cta, lane, a0, a1, at0);
                    const bool meets = lane < NW && a1 > a0 && a0 < (l + 1) * nbx && a1 > l * nbx;
                    const int contrib = __popc(__ballot_sync(0xffffffffu, meets));
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) {
                        __threadfence_block();
                        last = (atomicAdd(&red_cnt[l], 1) == contrib - 1);
                    }
                    last = __shfl_sync(0xffffffffu, last, 0);
                    if (last) {
                        __threadfence_block();
                        for (int i = lane; i < kRows * M; i += 32) {
                            const int row = i / M, m = i - row * M;
                            float *rp = red + (l * kRows + row) * kMP + m;
                            if (!dead)
                                Y[(int64_t)m * N + tile * kRows + row] = __float2half_rn(*rp);
                            *rp = 0.f;
                        }
                        if (lane == 0)
                            red_cnt[l] = 0;
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; e++) acc[e >> 3][(e >> 2) & 1][e & 3] = 0.f;
                from0 = true;
            }
            if (++box == nbx) { box = 0; ++tile; }
        }
        if (dead && lane == 0)
            flags[0] = 1;
        if (j == p.ntasks - 1)
            pdl_launch_dependents();
        __syncthreads();   // every Y store of task j in this CTA precedes its count
        if (flags[0]) {
            if (tid == ctl)
                atomicExch(p.cnt + p.ntasks, 1u);
            break;
        }
        if (tid == ctl) {
            // release: this CTA's Y stores of task j (ordered before this thread
            // by the barrier above) are visible before its count is.  This warp
            // issues no copies, so the release waits for nothing else.
            if (j < p.ntasks - 1) {
                if (j != p.withhold)
                    red_release_gpu(p.cnt + j, 1u);
            } else if (atom_add_acq_rel_gpu(p.cnt + j, 1u) == grid - 1) {
                for (int i = 0; i < p.ntasks; i++)   // every CTA is past its last wait
                    p.cnt[i] = 0u;
            }
        }
        // the deferred requests, while the control thread waits for the next task
        if (!control && !dead)
            refill(p.ntasks);
    }

    // after an abort: let the copies still in flight land before exiting
    if (!control && lane == 0) {
        for (int q = ccount; q < icount; q++) {
            const uint32_t bar = my_bars + 8 * (q % D);
            const unsigned long long tw = globaltimer();
            while (!mbar_try_wait(bar, (uint32_t)((q / D) & 1)) && globaltimer() - tw < kWaitLimitNs) {
            }
        }
    }
}

size_t smem_bytes(int nw, int depth, int M, int xs_stride, int ntasks) {
    return 1024 + (size_t)nw * depth * (kBoxBytes + kParBytes + 8) + (size_t)ntasks * sizeof(TaskInfo) +
           (size_t)M * xs_stride + 512 + (size_t)kMaxSplitTiles * kRows * kMP * 4 + 128;
}

constexpr size_t kSmemLimit = 227 * 1024;

template <bool BS64, bool ZP>
int launch_chain_t(const ChainHeader &h, const ChainParams &p, unsigned flags, cudaStream_t s) {
    auto fn = gemv_chain_kernel<BS64, ZP>;
    static int configured[kMaxDevices] = {};
    {
        cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(fn), h.smem, configured);
        if (e != cudaSuccess)
            return fail(MNB_ERR_CUDA, "mnb_gemv_chain: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    // every CTA waits for all others: the grid must be resident at once
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, (h.nw + 1) * 32, (size_t)h.smem);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv_chain: occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1 || per_sm * device_sm_count() < h.grid)
        return fail(MNB_ERR_UNSUPPORTED, "mnb_gemv_chain: %d CTAs of %d bytes cannot be resident together", h.grid,
                    h.smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)h.grid, 1, 1);
    cfg.blockDim = dim3((unsigned)((h.nw + 1) * 32), 1, 1);
    cfg.dynamicSmemBytes = (size_t)h.smem;
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
    e = cudaLaunchKernelEx(&cfg, fn, p);
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_gemv_chain: launch: %s", cudaGetErrorString(e));
    return MNB_OK;
}

}  // namespace

// Fault injection for tests (mnb_test_chain_withhold): read at each launch.
static int g_withhold = -1;
static unsigned long long g_task_wait_ns = kWaitLimitNs;

size_t gemv_chain_plan_bytes(int ntasks) {
    if (ntasks < 1 || ntasks > 65536)
        return 0;
    return sizeof(ChainHeader) + (size_t)ntasks * sizeof(ChainTask);
}

size_t gemv_chain_workspace_bytes(int ntasks) {
    if (ntasks < 1 || ntasks > 65536)
        return 0;
    return (((size_t)ntasks + 1) * sizeof(unsigned) + 255) / 256 * 256;
}

int gemv_chain_plan(const mnb_gemv_task *tasks, int ntasks, int M, int bs, void *plan, size_t plan_bytes) {
    static const char *fn = "mnb_gemv_chain_plan";
    const int has_zp = tasks[0].zp != nullptr;
    int nbx_max = 0;
    for (int j = 0; j < ntasks; j++) {
        const mnb_gemv_task &t = tasks[j];
        if (!t.X || !t.packed || !t.scales || !t.Y)
            return fail(MNB_ERR_INVALID_ARG, "%s: task %d has a NULL buffer", fn, j);
        if ((t.zp != nullptr) != (has_zp != 0))
            return fail(MNB_ERR_UNSUPPORTED, "%s: task %d: zero points present in some tasks only", fn, j);
        if (t.reserved != 0)
            return fail(MNB_ERR_INVALID_ARG, "%s: task %d: reserved field must be 0", fn, j);
        if (t.N < 16 || t.N % 16 != 0 || t.N > ((int64_t)1 << 28))
            return fail(MNB_ERR_SHAPE, "%s: task %d: N=%lld is not a positive multiple of 16 below 2^28", fn, j,
                        (long long)t.N);
        if (t.K < 256 || t.K % 256 != 0 || t.K > 65536 || (bs == 64 && has_zp && t.K % 512 != 0))
            return fail(MNB_ERR_SHAPE, "%s: task %d: K=%lld is not a multiple of %d in [256, 65536]", fn, j,
                        (long long)t.K, (bs == 64 && has_zp) ? 512 : 256);
        if (!aligned(t.X, 16) || !aligned(t.packed, 16) || !aligned(t.scales, bs == 32 ? 16 : 8) ||
            (has_zp && !aligned(t.zp, 4)) || !aligned(t.Y, 2))
            return fail(MNB_ERR_ALIGN, "%s: task %d: misaligned buffer", fn, j);
        nbx_max = std::max(nbx_max, (int)(t.K / kBoxK));
    }
    const int xs_stride = nbx_max * 512 + 64;
    // as many compute warps as fit with a ring of at least two slots each, then
    // the deepest ring that fits
    int depth = 0, nw = 0;
    for (int w = kMaxWarps; w >= 7 && !depth; w -= 4)
        for (int d = kMaxDepth; d >= 2 && !depth; d--)
            if (smem_bytes(w, d, M, xs_stride, ntasks) <= kSmemLimit) {
                depth = d;
                nw = w;
            }
    if (!depth)
        return fail(MNB_ERR_SHAPE, "%s: %d tasks at M=%d with K up to %d do not fit in shared memory", fn, ntasks, M,
                    nbx_max * kBoxK);
    EncodeTiledFn encode = tensor_map_encoder();
    if (!encode)
        return fail(MNB_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", fn);

    ChainHeader *hd = static_cast<ChainHeader *>(plan);
    ChainTask *out = reinterpret_cast<ChainTask *>(static_cast<unsigned char *>(plan) + sizeof(ChainHeader));
    memset(plan, 0, plan_bytes);
    const int grid = device_sm_count();
    int dev = 0;
    cudaGetDevice(&dev);
    hd->magic = kPlanMagic;
    hd->version = kPlanVersion;
    hd->ntasks = ntasks;
    hd->M = M;
    hd->bs = bs;
    hd->has_zp = has_zp;
    hd->grid = grid;
    hd->depth = depth;
    hd->xs_stride = xs_stride;
    hd->smem = (int)smem_bytes(nw, depth, M, xs_stride, ntasks);
    hd->nw = nw;
    hd->device = dev;
    for (int j = 0; j < ntasks; j++) {
        const mnb_gemv_task &t = tasks[j];
        ChainTask &o = out[j];
        const cuuint64_t gdim[2] = {(cuuint64_t)(t.K / 2), (cuuint64_t)t.N};
        const cuuint64_t gstride[1] = {(cuuint64_t)(t.K / 2)};
        const cuuint32_t box[2] = {128, (cuuint32_t)kRows};
        const cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&o.wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(t.packed), gdim,
                             gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS)
            return fail(MNB_ERR_CUDA, "%s: task %d: cuTensorMapEncodeTiled failed (%d)", fn, j, (int)cr);
        o.X = static_cast<const __half *>(t.X);
        o.scales = static_cast<const uint8_t *>(t.scales);
        o.zp = t.zp;
        o.Y = static_cast<__half *>(t.Y);
        o.N = (int)t.N;
        o.K = (int)t.K;
        o.nb = (int)(t.K / bs);
        o.zpb = (o.nb + 1) / 2;
        o.ntiles = o.N / kRows;
        o.nbx = o.K / kBoxK;
        o.tq = o.ntiles / grid;
        o.tr = o.ntiles % grid;
        o.wait = t.wait != 0;
    }
    return MNB_OK;
}

int launch_gemv_chain(const void *plan, const void *plan_device, void *workspace, size_t ws_bytes, unsigned flags,
                      cudaStream_t s) {
    static const char *fn = "mnb_gemv_chain";
    const ChainHeader &h = *static_cast<const ChainHeader *>(plan);
    if (h.magic != kPlanMagic || h.version != kPlanVersion || h.ntasks < 1 || h.ntasks > 65536)
        return fail(MNB_ERR_INVALID_ARG, "%s: not a plan written by mnb_gemv_chain_plan", fn);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != h.device)
        return fail(MNB_ERR_INVALID_ARG, "%s: plan made for device %d, current device is %d", fn, h.device, dev);
    if (ws_bytes < gemv_chain_workspace_bytes(h.ntasks))
        return fail(MNB_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, ws_bytes,
                    gemv_chain_workspace_bytes(h.ntasks));
    ChainParams p;
    p.tasks = reinterpret_cast<const ChainTask *>(static_cast<const unsigned char *>(plan_device) + sizeof(ChainHeader));
    p.cnt = static_cast<unsigned *>(workspace);
    p.ntasks = h.ntasks;
    p.M = h.M;
    p.depth = h.depth;
    p.xs_stride = h.xs_stride;
    p.nw = h.nw;
    p.withhold = (g_withhold < h.ntasks - 1) ? g_withhold : -1;   // the last task's count resets the counters
    p.task_wait_ns = g_task_wait_ns;
    if (h.nw < 7 || h.nw > kMaxWarps || h.depth < 2 || h.depth > kMaxDepth)
        return fail(MNB_ERR_INVALID_ARG, "%s: corrupt plan header", fn);
    if (h.bs == 64) {
        if (h.has_zp) return launch_chain_t<true, true>(h, p, flags, s);
        return launch_chain_t<true, false>(h, p, flags, s);
    }
    if (h.has_zp) return launch_chain_t<false, true>(h, p, flags, s);
    return launch_chain_t<false, false>(h, p, flags, s);
}

int read_chain_status(unsigned *out, int clear) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_chain_status, sizeof(unsigned));
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_chain_status, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return fail(MNB_ERR_CUDA, "mnb_device_status: %s", cudaGetErrorString(e));
    *out |= v << 1;   // bits 1 (a weight copy), 2 (a task's inputs), 3 (a workspace left dirty)
    return MNB_OK;
}

}  // namespace mnb

// Test hook: every later mnb_gemv_chain launch on any thread withholds the
// completion count of task `task` (-1: none; the last task's count is never
// withheld) and gives up a wait for a task's inputs after wait_limit_us
// microseconds (0: the default 2 s).  Declared in mnb_tune.h.
extern "C" MNB_API int mnb_test_chain_withhold(int task, int wait_limit_us) {
    if (task < -1 || wait_limit_us < 0 || wait_limit_us > 2000000)
        return MNB_ERR_INVALID_ARG;
    mnb::g_withhold = task;
    mnb::g_task_wait_ns = wait_limit_us ? (unsigned long long)wait_limit_us * 1000ull : mnb::kWaitLimitNs;
    return MNB_OK;
}
