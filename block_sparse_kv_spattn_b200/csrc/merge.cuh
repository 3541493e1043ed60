// merge.cuh -- the split merge: one softmax per output row from the partial
// records the attention kernels write per (CTA, unit) slot.
//
// "CSA + HCA 混合注意力机制" §4.4 step 4 (one softmax over the selected entries):
// a unit whose kept blocks were split over several CTAs gets partial results
// (base-2 maximum m_s, sum l_s, unnormalised output o_s per row), combined as
// out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#pragma once

#include "attention.cuh"

namespace spattn {

// A 16-byte global load issued here (the compiler may not sink it towards
// its use), so that several can be in flight before their results matter.
__device__ __forceinline__ float4 ld_f4_now(const float *p) {
    float4 v;
    asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}

struct MergeArgs {
    const float *part_o;
    const float *part_ml;
    const int32_t *sel_count;
    float *out;                 // [B][Tq][Hq][D]
    float *lse;                 // nullable: [B][Tq][Hq], ln of the row's sum of exp(logit)
    int batch, tq, hq, hkv, group, rows, units, max_sel, ctas;
    int ntiles;                 // row tiles (units) per (request, KV head); rows = rows of one tile
    int wslots;                 // partial records per (CTA, unit): 1 (attn_tcw, bf16), 2 (attn_tcw, fp8: two softmax halves) or 4 (one per attn_tc softmax warp)
    int pairs;                  // 4 records: warp w's pair w / 2 took only tiles of its parity
};

constexpr int kMergeMaxWarps = 16;  // warps per output row, for units split over many CTAs

// Records whose rows a warp loads together: 16, or 20 with the most warps
// (a unit spread over the whole grid, about 300 records, in one round).
__host__ __device__ constexpr int merge_group(int nw) { return nw >= kMergeMaxWarps ? 20 : 16; }

// Record x of a unit's candidate list (CTA c_lo + x / wslots, warp x %
// wslots), or -1 if it was not written: the CTA's range misses the unit's
// [pre, pre + cnt) part (only when W < C), or, with one record per
// tensor-core softmax warp, the warp's pair took none of the CTA's tiles of
// the unit (pair p takes CTA-local tile indices of parity p).
__host__ __device__ __forceinline__ int64_t merge_record(const MergeArgs &a, int x, int c_lo, int unit,
                                                         int64_t pre, int cnt, int64_t W) {
    const int cc = c_lo + x / a.wslots, w = x % a.wslots;
    const int64_t lo_c = W * cc / a.ctas, hi_c = W * (cc + 1) / a.ctas;
    const int64_t ia = (pre > lo_c ? pre : lo_c) - lo_c;
    const int64_t ib = (pre + cnt < hi_c ? pre + cnt : hi_c) - lo_c;
    if (ib <= ia) return -1;
    if (a.pairs && ib - ia < 2 && (ia & 1) != (w >> 1)) return -1;
    return ((int64_t)cc + unit) * a.wslots + w;
}

// One CTA of NW warps per output row (b, t, query head): out = sum_s
// 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the partial records of the
// row's unit: slot c + unit for each CTA c whose range meets the unit's part
// of the sequence (with wslots = 4, record w of that slot for each softmax
// warp w whose pair took one of the CTA's tiles of the unit: pair w / 2
// takes the tiles with CTA-local index of its parity).  The warps take
// groups of 16 records in turn (20 with 16 warps; a unit split over many
// CTAs has hundreds), each group's rows loaded together, and are combined
// through shared memory.  A unit with nothing kept gets a zero row.
//
// Launched early behind the attention kernel (programmatic dependent
// launch), which lets it be scheduled only once the selection is final: the
// unit's place in the concatenated sequence and the warp's first records
// are worked out from the selection counts before the wait (and their lines
// prefetched), the records themselves are read after it.
template <int NW>
__global__ void __launch_bounds__(NW * 32) merge_kernel(MergeArgs a) {
    constexpr int kMergeGroup = merge_group(NW);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t grow = blockIdx.x;
    const int i = (int)(grow % a.hq);
    const int t = (int)((grow / a.hq) % a.tq);
    const int b = (int)(grow / ((int64_t)a.hq * a.tq));
    const int h = i / a.group, g = i % a.group;
    const int rg = t * a.group + g;                 // the row in the chunk's Tq * group
    const int unit = (b * a.hkv + h) * a.ntiles + rg / a.rows;
    const int row = rg % a.rows;
    // prefix of the unit in the concatenated sequence, and the total W (four
    // count loads per lane in flight at a time)
    int64_t pre = 0, W = 0;
    for (int u0 = 0; u0 < a.units; u0 += 128) {
        int c4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int u = u0 + 32 * e + lane;
            c4[e] = u < a.units ? a.sel_count[a.ntiles == 1 ? u : u / a.ntiles] : 0;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int cnt = min(max(c4[e], 0), a.max_sel);
            W += cnt;
            if (u0 + 32 * e + lane < unit) pre += cnt;
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        pre += __shfl_xor_sync(0xffffffffu, pre, o);
        W += __shfl_xor_sync(0xffffffffu, W, o);
    }
    const int cnt = min(max(a.sel_count[unit / a.ntiles], 0), a.max_sel);
    // records r = (slot * wslots + w) that were written: CTAs with an empty
    // range (only when W < C) wrote none; with wslots = 4 a pair wrote only
    // if it took a tile
    int c_lo = 0, nrec = 0;
    if (cnt > 0) {
        c_lo = cta_of(pre, W, a.ctas);
        nrec = (cta_of(pre + cnt - 1, W, a.ctas) - c_lo + 1) * a.wslots;
    }
    int x0 = warp * kMergeGroup;
    int64_t r = lane < kMergeGroup && x0 + lane < nrec ? merge_record(a, x0 + lane, c_lo, unit, pre, cnt, W) : -1;
    // the records' lines (and translations) and the output row, before the wait
    for (int xp = x0; xp < nrec; xp += NW * kMergeGroup) {
        const int64_t rp = xp == x0 ? r : (lane < kMergeGroup && xp + lane < nrec
                                               ? merge_record(a, xp + lane, c_lo, unit, pre, cnt, W) : -1);
        if (rp >= 0) {
            prefetch_l2(a.part_o + (rp * a.rows + row) * kHeadDim);
            prefetch_l2(a.part_ml + (rp * a.rows + row) * 2);
        }
    }
    if (warp == 0 && lane == 31) prefetch_l2(a.out + grow * kHeadDim);
    asm volatile("griddepcontrol.wait;" ::: "memory");

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f, M = -INFINITY;
    for (; x0 < nrec; x0 += NW * kMergeGroup) {
        if (x0 != warp * kMergeGroup)
            r = lane < kMergeGroup && x0 + lane < nrec ? merge_record(a, x0 + lane, c_lo, unit, pre, cnt, W) : -1;
        const unsigned written = __ballot_sync(0xffffffffu, r >= 0);
        if (!written) continue;   // uniform
        // A written record's row is finite even when its maximum is -inf
        // (zero weights over zeroed unfilled slots), so the group's rows are
        // loaded together with the maxima, before the weights are known; a
        // record that was not written reads a written one (weight 0).
        const int64_t rfirst = __shfl_sync(0xffffffffu, r, __ffs(written) - 1);
        const int64_t rr = r >= 0 ? r : rfirst;
        const int n_here = nrec - x0 < kMergeGroup ? nrec - x0 : kMergeGroup;
        float4 o16[kMergeGroup];
#pragma unroll
        for (int e = 0; e < kMergeGroup; ++e) {
            const int64_t re = __shfl_sync(0xffffffffu, rr, e);
            o16[e] = e < n_here ? ld_f4_now(a.part_o + (re * a.rows + row) * kHeadDim + lane * 4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float2 ml = make_float2(-INFINITY, 0.f);
        if (r >= 0) ml = *reinterpret_cast<const float2 *>(a.part_ml + (r * a.rows + row) * 2);
        const float Mb = fmaxf(M, warp_max(ml.x));
        const unsigned valid = __ballot_sync(0xffffffffu, r >= 0 && ml.x != -INFINITY);
        if (valid && Mb != M) {   // uniform: rescale what is summed so far
            const float f = M == -INFINITY ? 0.f : exp2f(M - Mb);
            acc.x *= f;
            acc.y *= f;
            acc.z *= f;
            acc.w *= f;
            lsum *= f;
            M = Mb;
        }
        float w = 0.f;
        if ((valid >> lane) & 1u) {
            w = exp2f(ml.x - M);
            lsum = fmaf(w, ml.y, lsum);
        }
#pragma unroll
        for (int e = 0; e < kMergeGroup; ++e) {
            const float we = __shfl_sync(0xffffffffu, w, e);
            acc.x = fmaf(we, o16[e].x, acc.x);
            acc.y = fmaf(we, o16[e].y, acc.y);
            acc.z = fmaf(we, o16[e].z, acc.z);
            acc.w = fmaf(we, o16[e].w, acc.w);
        }
    }
    lsum = warp_sum(lsum);
    if constexpr (NW > 1) {
        // combine the warps: weights 2^(M_w - M)
        __shared__ float s_m[NW], s_l[NW];
        __shared__ float4 s_acc[NW][32];
        if (lane == 0) {
            s_m[warp] = M;
            s_l[warp] = lsum;
        }
        s_acc[warp][lane] = acc;
        __syncthreads();
        if (warp != 0) return;
        float Mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) Mt = fmaxf(Mt, s_m[w]);
        M = Mt;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        lsum = 0.f;
        if (Mt != -INFINITY)
            for (int w = 0; w < NW; ++w) {
                if (s_m[w] == -INFINITY) continue;
                const float f = exp2f(s_m[w] - Mt);
                const float4 o = s_acc[w][lane];
                lsum = fmaf(f, s_l[w], lsum);
                acc.x = fmaf(f, o.x, acc.x);
                acc.y = fmaf(f, o.y, acc.y);
                acc.z = fmaf(f, o.z, acc.z);
                acc.w = fmaf(f, o.w, acc.w);
            }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    reinterpret_cast<float4 *>(a.out + grow * kHeadDim)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    // records hold base-2 maxima of the scaled logits: ln sum = (M + log2 l) ln 2
    if (a.lse && lane == 0) a.lse[grow] = lsum > 0.f ? (M + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace spattn
