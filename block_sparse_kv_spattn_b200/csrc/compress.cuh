// compress.cuh -- mean-pooled key per (page, KV head).
//
// "Claude Code压缩上下文窗口的底层原理与性能优化实践", 算法流程 (均值池化合并):
// a run of tokens is merged into one vector by averaging; "CSA + HCA
// 混合注意力机制" §4.1 names plain averaging as the parameter-free compressor.
// Here the run is one 64-token block and the vector is the block's keys.
#pragma once

#include "common.cuh"

namespace spattn {

struct CompressArgs {
    const uint8_t *k_cache;   // bf16 or e4m3 bytes [num_pages][Hkv][P][D]
    const float *k_scale;     // [num_pages][Hkv] (fp8 only)
    const int32_t *block_table;
    const int32_t *old_lens;  // nullable
    const int32_t *seq_lens;
    void *kbar;               // [num_pages][Hkv][D] fp32, or bf16 when kbar_bf16
    int hkv, num_pages, max_blocks, kbar_bf16;
};

// Token groups per CTA so that a CTA has up to 512 threads.
__host__ __device__ constexpr int compress_groups(int hkv) {
    return 512 / (hkv * 16) < 8 ? 512 / (hkv * 16) : 8;
}

// Grid (gx, B); block = TG * Hkv * 16 threads: thread (g, h, chunk) sums 8
// columns of KV head h over the tokens t = g, g + TG, ... of a block (all its
// loads issued together), and the TG partial sums are added in a fixed order
// through shared memory.  CTA x walks the touched blocks of request y with
// stride gx.
template <bool FP8, int TG>
__global__ void __launch_bounds__(512) compress_keys_kernel(CompressArgs a) {
    constexpr int TPG = kBlock / TG;  // tokens per group
    extern __shared__ float4 part4[];  // [TG][Hkv*16][2] float4
    const int b = blockIdx.y;
    const int lanes = a.hkv * 16;
    const int hc = threadIdx.x % lanes, g = threadIdx.x / lanes;
    const int h = hc >> 4, chunk = hc & 15;
    const int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(SPATTN_DEV_BAD_LEN);
        return;
    }
    const int nb = (L + kBlock - 1) / kBlock;
    int j_lo = 0;
    if (a.old_lens) {
        int o = a.old_lens[b];
        o = o < 0 ? 0 : (o > L ? L : o);
        j_lo = o / kBlock;
        if (o == L) return;  // nothing appended
    }
    for (int j = j_lo + blockIdx.x; j < nb; j += gridDim.x) {
        const int page = a.block_table[(int64_t)b * a.max_blocks + j];
        if (page < 0 || page >= a.num_pages) {
            if (threadIdx.x == 0) flag(SPATTN_DEV_BAD_PAGE);
            continue;
        }
        const int filled = min(kBlock, L - j * kBlock);
        const int64_t tile = ((int64_t)page * a.hkv + h) * kBlock * kHeadDim;
        float s[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) s[c] = 0.f;
#pragma unroll
        for (int k = 0; k < TPG; ++k) {
            const int t = g + k * TG;
            if (t < filled) {
                float f[8];
                if (FP8) {
                    const uint2 u = *reinterpret_cast<const uint2 *>(a.k_cache + tile + t * kHeadDim + chunk * 8);
                    e4m3x8_to_f32(u, f);
                } else {
                    const uint4 u = *reinterpret_cast<const uint4 *>(a.k_cache + 2 * (tile + t * kHeadDim + chunk * 8));
                    bf16x8_to_f32(u, f);
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) s[c] += f[c];
            }
        }
        part4[(g * lanes + hc) * 2 + 0] = make_float4(s[0], s[1], s[2], s[3]);
        part4[(g * lanes + hc) * 2 + 1] = make_float4(s[4], s[5], s[6], s[7]);
        __syncthreads();
        if (g == 0) {
            float4 x = part4[hc * 2], y = part4[hc * 2 + 1];
#pragma unroll
            for (int gg = 1; gg < TG; ++gg) {
                const float4 u = part4[(gg * lanes + hc) * 2], v = part4[(gg * lanes + hc) * 2 + 1];
                x.x += u.x; x.y += u.y; x.z += u.z; x.w += u.w;
                y.x += v.x; y.y += v.y; y.z += v.z; y.w += v.w;
            }
            const float sc = FP8 ? a.k_scale[(int64_t)page * a.hkv + h] : 1.f;
            const float n = (float)filled;
            const int64_t at = ((int64_t)page * a.hkv + h) * kHeadDim + chunk * 8;
            const float m[8] = {x.x * sc / n, x.y * sc / n, x.z * sc / n, x.w * sc / n,
                                y.x * sc / n, y.y * sc / n, y.z * sc / n, y.w * sc / n};
            if (a.kbar_bf16) {
                // the fp32 mean rounded to bf16 (nearest even)
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 v = __floats2bfloat162_rn(m[2 * e], m[2 * e + 1]);
                    w[e] = *reinterpret_cast<const uint32_t *>(&v);
                }
                *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.kbar) + at) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.kbar) + at);
                dst[0] = make_float4(m[0], m[1], m[2], m[3]);
                dst[1] = make_float4(m[4], m[5], m[6], m[7]);
            }
        }
        __syncthreads();
    }
}

}  // namespace spattn
