// hca.cuh -- the weight-free HCA branch: pooled entries and dense attention
// over them, and the log-sum-exp merge with the sparse branch.
//
// "CSA + HCA 混合注意力机制" §5.1-5.2: every m' = 128 consecutive tokens become
// one entry; each query attends over all entries with no selection.  Mean
// pooling stands in for the page's learned pooling; an entry is visible to a
// query once all its tokens are at or before the query's position; no
// position tag and no sink logit (both learned).  The two branches' results
// combine by their log-sum-exp: softmax attention over both key sets.
#pragma once

#include "common.cuh"

namespace spattn {

constexpr int kHcaGroupBlocks = 2;                  // 128-token entries
constexpr int kHcaTokens = kHcaGroupBlocks * kBlock;
constexpr int kHcaWarps = 16;                       // warps per output row (attention)
constexpr int kHcaBatch = 4;                        // entries a warp loads at once

struct HcaPoolArgs {
    const uint8_t *k_cache, *v_cache;   // bf16 or e4m3 bytes [num_pages][Hkv][P][D]
    const float *k_scale, *v_scale;     // fp8 only
    const int32_t *block_table;
    const int32_t *old_lens;            // nullable: every entry
    const int32_t *seq_lens;
    float *khat, *vhat;                 // [B][G_max][Hkv][D]
    int hkv, num_pages, max_blocks, gmax;
};

// Grid (gx, B), Hkv warps: warp h sums K and V of KV head h over an entry's
// tokens (lane: 4 columns) in fp32, then divides by the token count; the
// CTAs stride over the entries.  Without old_lens every entry is written
// (zeros past the end of the request); with old_lens only the entries that
// hold a token of [old_len, L).
template <bool FP8>
__global__ void __launch_bounds__(16 * 32) hca_pool_kernel(HcaPoolArgs a) {
    const int b = blockIdx.y, h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (h >= a.hkv) return;
    const int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(SPATTN_DEV_BAD_LEN);
        return;
    }
    int g_lo = 0, g_hi = a.gmax;
    if (a.old_lens) {
        g_lo = min(max(a.old_lens[b], 0), L) / kHcaTokens;
        g_hi = (L + kHcaTokens - 1) / kHcaTokens;
    }
    for (int g = g_lo + blockIdx.x; g < g_hi; g += gridDim.x) {
        const int t0 = g * kHcaTokens, t1 = min(L, t0 + kHcaTokens);
        float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
        for (int blk = 0; blk < kHcaGroupBlocks && t0 + blk * kBlock < t1; ++blk) {
            const int j = g * kHcaGroupBlocks + blk;
            const int page = a.block_table[(int64_t)b * a.max_blocks + j];
            if (page < 0 || page >= a.num_pages) {
                if (lane == 0) flag(SPATTN_DEV_BAD_PAGE);
                continue;
            }
            const int n = min(kBlock, t1 - j * kBlock);
            const int64_t base = ((int64_t)page * a.hkv + h) * kBlock * kHeadDim + lane * 4;
            float ksc = 1.f, vsc = 1.f;
            if (FP8) {
                ksc = a.k_scale[(int64_t)page * a.hkv + h];
                vsc = a.v_scale[(int64_t)page * a.hkv + h];
            }
            float4 bk = make_float4(0.f, 0.f, 0.f, 0.f), bv = bk;
#pragma unroll 4
            for (int t = 0; t < n; ++t) {
                float kx[4], vx[4];
                if (FP8) {
                    const uint32_t ku = *reinterpret_cast<const uint32_t *>(a.k_cache + base + t * kHeadDim);
                    const uint32_t vu = *reinterpret_cast<const uint32_t *>(a.v_cache + base + t * kHeadDim);
                    e4m3x2_to_f32((uint16_t)(ku & 0xffffu), kx[0], kx[1]);
                    e4m3x2_to_f32((uint16_t)(ku >> 16), kx[2], kx[3]);
                    e4m3x2_to_f32((uint16_t)(vu & 0xffffu), vx[0], vx[1]);
                    e4m3x2_to_f32((uint16_t)(vu >> 16), vx[2], vx[3]);
                } else {
                    const uint2 ku = *reinterpret_cast<const uint2 *>(a.k_cache + (base + t * kHeadDim) * 2);
                    const uint2 vu = *reinterpret_cast<const uint2 *>(a.v_cache + (base + t * kHeadDim) * 2);
                    kx[0] = bf16lo(ku.x), kx[1] = bf16hi(ku.x), kx[2] = bf16lo(ku.y), kx[3] = bf16hi(ku.y);
                    vx[0] = bf16lo(vu.x), vx[1] = bf16hi(vu.x), vx[2] = bf16lo(vu.y), vx[3] = bf16hi(vu.y);
                }
                bk.x += kx[0], bk.y += kx[1], bk.z += kx[2], bk.w += kx[3];
                bv.x += vx[0], bv.y += vx[1], bv.z += vx[2], bv.w += vx[3];
            }
            sk.x = fmaf(bk.x, ksc, sk.x), sk.y = fmaf(bk.y, ksc, sk.y);
            sk.z = fmaf(bk.z, ksc, sk.z), sk.w = fmaf(bk.w, ksc, sk.w);
            sv.x = fmaf(bv.x, vsc, sv.x), sv.y = fmaf(bv.y, vsc, sv.y);
            sv.z = fmaf(bv.z, vsc, sv.z), sv.w = fmaf(bv.w, vsc, sv.w);
        }
        const float inv = t1 > t0 ? 1.f / (float)(t1 - t0) : 0.f;
        const int64_t o = (((int64_t)b * a.gmax + g) * a.hkv + h) * kHeadDim + lane * 4;
        *reinterpret_cast<float4 *>(a.khat + o) = make_float4(sk.x * inv, sk.y * inv, sk.z * inv, sk.w * inv);
        *reinterpret_cast<float4 *>(a.vhat + o) = make_float4(sv.x * inv, sv.y * inv, sv.z * inv, sv.w * inv);
    }
}

struct HcaAttendArgs {
    const uint16_t *q;          // bf16 bits [B][Tq][Hq][D]
    const float *khat, *vhat;   // [B][G_max][Hkv][D]
    const int32_t *seq_lens;
    float *out;                 // [B][Tq][Hq][D]
    float *lse;                 // [B][Tq][Hq], natural log
    int tq, hq, hkv, max_blocks, gmax;
    float qscale;               // sm_scale * log2(e)
};

// One CTA per output row (b, t, query head), kHcaWarps warps, each taking a
// contiguous slice of the visible entries with an online softmax (base 2,
// lane: 4 columns); the warps combine through shared memory.
__global__ void __launch_bounds__(kHcaWarps * 32) hca_attend_kernel(HcaAttendArgs a) {
    __shared__ float s_m[kHcaWarps], s_l[kHcaWarps];
    __shared__ float4 s_acc[kHcaWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int i = (int)(row % a.hq), t = (int)((row / a.hq) % a.tq), b = (int)(row / ((int64_t)a.hq * a.tq));
    const int h = i / (a.hq / a.hkv);
    int L = a.seq_lens[b];
    L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
    const int qpos = L - a.tq + t;
    // visible entries: all tokens at or before qpos
    const int ng = qpos < 0 ? 0 : min((qpos + 1) / kHcaTokens + (qpos + 1 == L && L % kHcaTokens ? 1 : 0),
                                      (L + kHcaTokens - 1) / kHcaTokens);
    const uint2 qu = reinterpret_cast<const uint2 *>(a.q + row * kHeadDim)[lane];
    const float4 qv = make_float4(bf16lo(qu.x) * a.qscale, bf16hi(qu.x) * a.qscale, bf16lo(qu.y) * a.qscale,
                                  bf16hi(qu.y) * a.qscale);
    const int lo = (int)((int64_t)ng * warp / kHcaWarps), hi = (int)((int64_t)ng * (warp + 1) / kHcaWarps);
    const float4 *kp = reinterpret_cast<const float4 *>(a.khat) + ((int64_t)b * a.gmax * a.hkv + h) * 32 + lane;
    const float4 *vp = reinterpret_cast<const float4 *>(a.vhat) + ((int64_t)b * a.gmax * a.hkv + h) * 32 + lane;
    const int64_t gstride = (int64_t)a.hkv * 32;   // float4s from one entry to the next
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // kHcaBatch entries at a time: their loads and dot products overlap, one
    // rescale per batch
    for (int g = lo; g < hi; g += kHcaBatch) {
        const int n = min(kHcaBatch, hi - g);
        float4 k[kHcaBatch], v[kHcaBatch];
        float s[kHcaBatch];
#pragma unroll
        for (int e = 0; e < kHcaBatch; ++e) {
            const int ge = e < n ? g + e : g;
            k[e] = kp[ge * gstride];
            v[e] = vp[ge * gstride];
        }
#pragma unroll
        for (int e = 0; e < kHcaBatch; ++e) {
            float x = qv.x * k[e].x;
            x = fmaf(qv.y, k[e].y, x);
            x = fmaf(qv.z, k[e].z, x);
            s[e] = fmaf(qv.w, k[e].w, x);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int e = 0; e < kHcaBatch; ++e) s[e] += __shfl_xor_sync(0xffffffffu, s[e], o);
        float mx = s[0];
#pragma unroll
        for (int e = 1; e < kHcaBatch; ++e) mx = e < n ? fmaxf(mx, s[e]) : mx;
        if (mx > m) {   // uniform: rescale what is summed so far
            const float f = exp2f(m - mx);
            l *= f;
            acc.x *= f, acc.y *= f, acc.z *= f, acc.w *= f;
            m = mx;
        }
#pragma unroll
        for (int e = 0; e < kHcaBatch; ++e) {
            const float p = e < n ? exp2f(s[e] - m) : 0.f;
            l += p;
            acc.x = fmaf(p, v[e].x, acc.x), acc.y = fmaf(p, v[e].y, acc.y);
            acc.z = fmaf(p, v[e].z, acc.z), acc.w = fmaf(p, v[e].w, acc.w);
        }
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
    s_acc[warp][lane] = acc;
    __syncthreads();
    if (warp != 0) return;
    float M = -INFINITY;
    for (int w = 0; w < kHcaWarps; ++w) M = fmaxf(M, s_m[w]);
    float lt = 0.f;
    float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY)
        for (int w = 0; w < kHcaWarps; ++w) {
            if (s_m[w] == -INFINITY) continue;
            const float f = exp2f(s_m[w] - M);
            const float4 x = s_acc[w][lane];
            lt = fmaf(f, s_l[w], lt);
            at.x = fmaf(f, x.x, at.x), at.y = fmaf(f, x.y, at.y), at.z = fmaf(f, x.z, at.z), at.w = fmaf(f, x.w, at.w);
        }
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    reinterpret_cast<float4 *>(a.out + row * kHeadDim)[lane] = make_float4(at.x * inv, at.y * inv, at.z * inv, at.w * inv);
    if (lane == 0) a.lse[row] = lt > 0.f ? (M + log2f(lt)) * 0.69314718055994531f : -INFINITY;
}

// out = (e^lse_a out_a + e^lse_b out_b) / (e^lse_a + e^lse_b) per row, one
// warp per row; lse = ln of the sum (rows with neither: 0 and -inf).  out
// and lse may be the same buffers as either input.
__global__ void __launch_bounds__(256) lse_merge_kernel(int64_t rows, const float *oa, const float *la,
                                                        const float *ob, const float *lb, float *out,
                                                        float *lse) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float A = la[row], B = lb[row];
    const float M = fmaxf(A, B);
    float wa = 0.f, wb = 0.f;
    if (M != -INFINITY) {
        wa = A == -INFINITY ? 0.f : expf(A - M);
        wb = B == -INFINITY ? 0.f : expf(B - M);
    }
    const float z = wa + wb, inv = z > 0.f ? 1.f / z : 0.f;
    const float4 x = reinterpret_cast<const float4 *>(oa + row * kHeadDim)[lane];
    const float4 y = reinterpret_cast<const float4 *>(ob + row * kHeadDim)[lane];
    __syncwarp();   // every lane has read la, lb: out and lse may alias the inputs
    reinterpret_cast<float4 *>(out + row * kHeadDim)[lane] =
        make_float4((wa * x.x + wb * y.x) * inv, (wa * x.y + wb * y.y) * inv, (wa * x.z + wb * y.z) * inv,
                    (wa * x.w + wb * y.w) * inv);
    if (lse && lane == 0) lse[row] = z > 0.f ? M + logf(z) : -INFINITY;
}

}  // namespace spattn
