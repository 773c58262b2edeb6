// common.cuh -- shared host/device helpers of libmnb (the CUDA side only).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mnb.h"

namespace mnb {

// ---------------------------------------------------------------- host errors

// Records a message for mnb_last_error() and returns `code`.
int fail(int code, const char *fmt, ...);
void clear_error();
// Maps a CUDA error from the launch just made to MNB_ERR_CUDA (or MNB_OK).
int check_launch(const char *what);

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// cuTensorMapEncodeTiled from the driver, or null when it is unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device when it is below that; `cache` (one entry per device, zero-initialized
// by the caller as a static array of kMaxDevices) remembers what each device
// was given.  Returns a cudaError_t.
constexpr int kMaxDevices = 128;
cudaError_t ensure_dynamic_smem(const void *kernel, int bytes, int *cache);

// ---------------------------------------------------------------- device PTX

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    // (a & mask) | magic in one instruction (truth table 0xEA).
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

// 16-byte streaming load that does not allocate in L1 (weights are read once).
// Read-only data for the whole kernel, so the asm is free to move.
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// 16-byte load served by L2 (not L1): for activations that the previous kernel
// in the stream may have just written.
__device__ __forceinline__ uint4 ldg_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Programmatic dependent launch controls (no-ops when launched without PDL).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bit casts between a 32-bit register and a half2 (memcpy: no aliasing games).
__device__ __forceinline__ half2 u32_as_h2(uint32_t v) {
    half2 h;
    memcpy(&h, &v, sizeof(h));
    return h;
}
__device__ __forceinline__ uint32_t h2_as_u32(half2 v) {
    uint32_t u;
    memcpy(&u, &v, sizeof(u));
    return u;
}

// ---- mbarrier, TMA and timer wrappers shared by the TMA-fed kernels --------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 2D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- cluster, MMA and int4 unpack helpers shared by the kernels ------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// D += A . B on the legacy tensor path: m16n8k16, fp16 inputs, fp32 accumulator.
__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 32-bit word of nibbles e0..e7 of a row -> the A-operand half2 (e0,e4),
// 16(e1,e5), (e2,e6), 16(e3,e7): (1024 + q) - (1024 + zp) = q - zp exactly,
// times the fp16 scale = fp16_rn((q - zp) * s) (x16 for the high nibbles, also
// exact).  Z = 1024 + zp and Zhi = 1024 + 16 zp as fp16 pairs.
__device__ __forceinline__ void dq_word(uint32_t w, uint32_t s2, uint32_t Z, uint32_t Zhi, uint32_t &a0,
                                        uint32_t &a1, uint32_t &a2, uint32_t &a3) {
    const uint32_t w8 = w >> 8;
    const half2 s = u32_as_h2(s2);
    a0 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s));
    a1 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), u32_as_h2(Zhi)), s));
    a2 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w8, 0x000F000Fu, 0x64006400u)), u32_as_h2(Z)), s));
    a3 = h2_as_u32(__hmul2(__hsub2(u32_as_h2(lop3_and_or(w8, 0x00F000F0u, 0x64006400u)), u32_as_h2(Zhi)), s));
}

}  // namespace mnb
