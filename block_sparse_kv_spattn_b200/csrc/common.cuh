// common.cuh -- device helpers shared by the spattn kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spattn.h"

namespace spattn {

constexpr int kHeadDim = 128;
constexpr int kBlock = 64;
constexpr float kLog2e = 1.4426950408889634f;

// Device status word: kernels OR SPATTN_DEV_* bits into it instead of
// trapping.  One instance per device (module-scope __device__ variable).
__device__ int32_t g_status;

__device__ __forceinline__ void flag(int32_t bits) { atomicOr(&g_status, bits); }

// ---------------------------------------------------------------- numbers

// Two packed bf16 -> two fp32 (bf16 is the high half of a binary32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x);
    f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z);
    f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}

// Two e4m3fn codes (low byte first) -> two fp32, through the hardware
// e4m3x2 -> f16x2 conversion (exact: every e4m3 value is an f16 value).
__device__ __forceinline__ void e4m3x2_to_f32(uint16_t codes, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
    __half2 hv = *reinterpret_cast<__half2 *>(&h2);
    float2 f = __half22float2(hv);
    lo = f.x;
    hi = f.y;
}

__device__ __forceinline__ void e4m3x8_to_f32(const uint2 &u, float (&f)[8]) {
    e4m3x2_to_f32((uint16_t)(u.x & 0xffff), f[0], f[1]);
    e4m3x2_to_f32((uint16_t)(u.x >> 16), f[2], f[3]);
    e4m3x2_to_f32((uint16_t)(u.y & 0xffff), f[4], f[5]);
    e4m3x2_to_f32((uint16_t)(u.y >> 16), f[6], f[7]);
}

// Order-preserving map float -> uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// ------------------------------------------------------------ mbarriers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of phase `parity` (never suspends the thread, unlike
// try_wait): for a thread that polls several barriers in turn.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete, giving up after ~1 s.
// Returns false (and sets SPATTN_DEV_WAIT_TIMEOUT) when it gave up.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            flag(SPATTN_DEV_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Bulk (non-tensor) async copy global -> shared, completion counted in bytes
// on `bar`.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------- reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive scan of an int over a warp.
// L2 prefetch of the line holding p.  It uses no data, so a kernel launched
// early may issue it before its wait on the kernel that writes p; its use is
// that p's address translation and line are in place when p is accessed.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__device__ __forceinline__ float warp_incl_scan_f(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Block-wide exclusive scan of one int per thread; `tmp` holds 32 ints of
// shared memory; returns the exclusive prefix, *total the block sum.
// Every thread of the block must call it.
__device__ __forceinline__ int block_excl_scan(int v, int *tmp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    int inc = warp_incl_scan(v);
    __syncthreads();
    if (lane == 31) tmp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? tmp[lane] : 0;
        int wi = warp_incl_scan(w);
        if (lane < nw) tmp[lane] = wi - w;
        if (lane == nw - 1) tmp[32] = wi;
    }
    __syncthreads();
    int res = inc - v + tmp[warp];
    *total = tmp[32];
    return res;
}

// Block-wide inclusive scan of one float per thread (same contract).
__device__ __forceinline__ float block_incl_scan_f(float v, float *tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    float inc = warp_incl_scan_f(v);
    __syncthreads();
    if (lane == 31) tmp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        float w = lane < nw ? tmp[lane] : 0.f;
        float wi = warp_incl_scan_f(w);
        if (lane < nw) tmp[lane] = wi - w;
    }
    __syncthreads();
    return inc + tmp[warp];
}

}  // namespace spattn
