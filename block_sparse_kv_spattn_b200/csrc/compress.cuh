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
    float *kbar;              // [num_pages][Hkv][D]
    int hkv, num_pages, max_blocks;
};

// Grid (gx, B); block = Hkv * 16 threads: thread (h, chunk) owns 8 columns
// of KV head h.  CTA x walks the touched blocks of request y with stride gx.
// Four interleaved fp32 partial sums per column keep the rounding error of
// the 64-term sum near that of a depth-5 tree.
template <bool FP8>
__global__ void compress_keys_kernel(CompressArgs a) {
    const int b = blockIdx.y;
    const int h = threadIdx.x >> 4, chunk = threadIdx.x & 15;
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
        float s[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int c = 0; c < 8; ++c) s[q][c] = 0.f;
        for (int t0 = 0; t0 < filled; t0 += 4) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = t0 + q;
                if (t < filled) {
                    float f[8];
                    if (FP8) {
                        uint2 u = *reinterpret_cast<const uint2 *>(a.k_cache + tile + t * kHeadDim +
                                                                   chunk * 8);
                        e4m3x8_to_f32(u, f);
                    } else {
                        uint4 u = *reinterpret_cast<const uint4 *>(
                            a.k_cache + 2 * (tile + t * kHeadDim + chunk * 8));
                        bf16x8_to_f32(u, f);
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) s[q][c] += f[c];
                }
            }
        }
        const float sc = FP8 ? a.k_scale[(int64_t)page * a.hkv + h] : 1.f;
        float r[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            r[c] = (((s[0][c] + s[1][c]) + (s[2][c] + s[3][c])) * sc) / (float)filled;
        float4 *dst = reinterpret_cast<float4 *>(a.kbar + ((int64_t)page * a.hkv + h) * kHeadDim +
                                                 chunk * 8);
        dst[0] = make_float4(r[0], r[1], r[2], r[3]);
        dst[1] = make_float4(r[4], r[5], r[6], r[7]);
    }
}

}  // namespace spattn
