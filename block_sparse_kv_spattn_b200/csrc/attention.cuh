// attention.cuh -- what the attention kernels share: their arguments, the
// balanced split of the kept blocks, the stage metadata, and the split merge.
//
// "CSA + HCA 混合注意力机制" §2.1 / §4.4 step 4: softmax(q K_sel^T / sqrt(d)) V_sel
// over the selected entries only; §4.3: the window blocks and the partly
// filled tail block join the same softmax.  §2.3: the decode step is bound by
// reading K and V from HBM.
//
// Work split (balanced, persistent): the kept lists of all (request, KV head)
// units are concatenated into one sequence of W blocks and CTA c of C takes
// blocks [c*W/C, (c+1)*W/C).  Each maximal run of one unit inside a CTA's
// range is a "segment"; the CTA writes partial records (running max in log2
// units, sum, unnormalised output per query row) per segment into slot
// c + unit, which is unique along the monotone (c, unit) staircase.
// merge.cuh combines the partials of a unit by their log-sum-exp.  The
// kernels themselves are attention_tc.cuh (bf16 caches, up to 16 query rows
// per KV head) and attention_tcw.cuh (up to 64 rows, bf16 or fp8 caches).
#pragma once

#include "common.cuh"

namespace spattn {

struct AttnArgs {
    const uint16_t *q;          // bf16 bits [B][Tq][Hq][D]
    const uint8_t *k_cache;     // [num_pages][Hkv][P][D] bf16 or e4m3 bytes
    const uint8_t *v_cache;
    const float *k_scale;       // fp8 only
    const float *v_scale;
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int32_t *sel_idx;     // [B*Hkv][max_sel]
    const int32_t *sel_count;   // [B*Hkv]
    float *part_o;              // [(C + units) * records per slot][rows][D]
    float *part_ml;             // [(C + units) * records per slot][rows][2]
    // rows: query rows per unit (Tq * group, at most 64 for attn_tcw_kernel);
    // a (request, KV head) with more query rows is split into ntiles units
    // of 64 rows, unit u = (b * hkv + h) * ntiles + tile, each over the same
    // kept blocks (the query-tile outer loop of flash attention)
    int tq, hq, hkv, group, rows, units, num_pages, max_blocks, max_sel;
    int ntiles, rows_total;     // row tiles per (request, KV head); Tq * group
    float qscale;               // sm_scale * log2(e)
};

struct StageMeta {
    int j;        // logical block id
    int page;     // page id, -1 when the block or its page is invalid
    int unit;     // (b * Hkv + h) * ntiles + row tile
    int flags;    // kFirst | kLast | kEnd
    int seg;      // segment id within the CTA (tensor-core kernel)
    int unused1;
    int qslot;    // query slot holding the segment's query rows
    int pad;
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

__host__ __device__ constexpr int align16(int x) { return (x + 15) / 16 * 16; }

__device__ __forceinline__ int unit_count(const AttnArgs &a, int u) {
    return min(max(a.sel_count[a.ntiles == 1 ? u : u / a.ntiles], 0), a.max_sel);
}

// CTA whose range [c*W/C, (c+1)*W/C) holds flattened index x (0 <= x < W).
__host__ __device__ __forceinline__ int cta_of(int64_t x, int64_t W, int C) {
    return (int)(((x + 1) * C + W - 1) / W) - 1;
}
}  // namespace spattn
