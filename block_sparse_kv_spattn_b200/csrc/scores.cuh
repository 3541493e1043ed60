// scores.cuh -- score every middle block against its compressed key.
//
// "CSA + HCA 混合注意力机制" §4.2 (Lightning Indexer, steps 3-4: every
// compressed entry gets a score from the query, heads are aggregated into one
// score per entry) and §4.4 step 1.  Without learned indexer projections the
// score of block j for KV head h is the mean of the group's per-head logits
// against the block's mean key: (qbar . kbar_j) * sm_scale, qbar the mean of
// the group's query rows.
#pragma once

#include "common.cuh"

namespace spattn {

struct ScoresArgs {
    const uint16_t *q;        // bf16 bits [B][Tq][Hq][D]
    const void *kbar;         // [num_pages][Hkv][D] fp32, or bf16 (KB16)
    const int32_t *block_table;
    const int32_t *seq_lens;
    float *scores;            // [B][Tq][Hkv][max_blocks]
    int tq, hq, num_pages, max_blocks, sink, local, bpc;
    int tt;                   // query tokens per CTA (grid z tiles a chunk's tokens)
    int anchors;              // also score the sink and local blocks (anchor-adaptive selection)
    float scale;
};

constexpr int kScoreThreads = 128;

// Blocks per CTA: small CTAs (many resident per SM, many loads in flight)
// unless the query rows make the per-CTA q-bar prologue heavy, or there are
// so few rows (one or two KV heads of a decode step) that a CTA's compressed
// keys are a short read beside its prologue.
__host__ __device__ constexpr int score_blocks_per_cta(int rows) { return rows <= 2 ? 64 : (rows <= 16 ? 16 : 64); }
static_assert(score_blocks_per_cta(1) <= kScoreThreads && score_blocks_per_cta(64) <= kScoreThreads,
              "one block-table entry per thread");

// Sum of v[0..7] over the 32 lanes, scattered: afterwards lane l holds the
// full sum of element (l >> 2) & 7.  Butterfly halving at offsets 16, 8, 4
// (each lane keeps the half named by its offset bit), then plain xor
// reductions at 2 and 1: 9 shuffles for 8 warp sums.
__device__ __forceinline__ float reduce_scatter8(float (&v)[8]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 3; ++step) {
        const int off = 16 >> step;
        const int half = 4 >> step;
        const bool up = lane & off;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            float send = up ? v[i] : v[i + half];
            float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float r = v[0];
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    return r;
}

// Lane's 4 columns of every KV head's compressed key of one page, as fp32
// (bf16 keys widened exactly).
template <int HKV, bool KB16>
__device__ __forceinline__ void load_kbar(const void *kbar, int page, int lane, float4 (&kv)[HKV]) {
    if (KB16) {
        const uint2 *kp =
            reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(kbar) + (int64_t)page * HKV * kHeadDim);
#pragma unroll
        for (int hh = 0; hh < HKV; ++hh) {
            const uint2 u = kp[hh * (kHeadDim / 4) + lane];
            kv[hh] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                 __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        }
    } else {
        const float4 *kp =
            reinterpret_cast<const float4 *>(static_cast<const float *>(kbar) + (int64_t)page * HKV * kHeadDim);
#pragma unroll
        for (int hh = 0; hh < HKV; ++hh) kv[hh] = kp[hh * (kHeadDim / 4) + lane];
    }
}

// Grid (ceil(max_blocks / bpc), B, ceil(Tq / tt)), kScoreThreads threads.
// Dynamic shared memory: qbar [tt][HKV][D] fp32, a [tt*HKV][bpc] output tile,
// then the page ids of the CTA's middle blocks (-1 elsewhere), read in the
// prologue alongside the query rows.
// Warp w takes blocks w, w + 4, ... of the CTA's range, BIF of them at a
// time with all their compressed-key loads issued together.
template <int HKV, bool KB16>
__global__ void __launch_bounds__(kScoreThreads, 5) block_scores_kernel(ScoresArgs a) {
    constexpr int BIF = HKV >= 16 ? 1 : (HKV >= 8 ? 2 : 4);
    constexpr int NW = kScoreThreads / 32;
    extern __shared__ float4 smem_f4[];
    float *qbar = reinterpret_cast<float *>(smem_f4);
    const int tb = blockIdx.z * a.tt;                 // this CTA's first query token
    const int ntok = min(a.tt, a.tq - tb);
    const int rows = ntok * HKV;
    float *tile = qbar + rows * kHeadDim;
    int *pages = reinterpret_cast<int *>(tile + rows * a.bpc);
    const int b = blockIdx.y;
    const int j0 = blockIdx.x * a.bpc;
    const int G = a.hq / HKV;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the selection grid that follows may be scheduled now: it waits for
    // this grid's completion before it reads the scores
    asm volatile("griddepcontrol.launch_dependents;");

    // this thread's block-table entry (one block of the CTA's range per
    // thread), loaded beside the length instead of after it: which entries
    // count is decided once the length is known
    const int tj = threadIdx.x, tblk = j0 + tj;
    const int page_raw =
        (tj < a.bpc && tblk < a.max_blocks) ? a.block_table[(int64_t)b * a.max_blocks + tblk] : -1;
    int L = a.seq_lens[b];
    // 1. group-mean query rows (8 columns per task); their loads, the length
    // and the table entry are in flight together
    for (int task = threadIdx.x; task < rows * (kHeadDim / 8); task += kScoreThreads) {
        const int c8 = task % (kHeadDim / 8), th = task / (kHeadDim / 8);
        const int hh = th % HKV, t = th / HKV;
        const uint16_t *qr = a.q + (((int64_t)b * a.tq + tb + t) * a.hq + hh * G) * kHeadDim + c8 * 8;
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int g0 = 0; g0 < G; g0 += 8) {  // the group's rows are loaded 8 at a time
            uint4 u[8];
#pragma unroll
            for (int gg = 0; gg < 8; ++gg)
                if (g0 + gg < G) u[gg] = *reinterpret_cast<const uint4 *>(qr + (g0 + gg) * kHeadDim);
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) {
                if (g0 + gg < G) {
                    float f[8];
                    bf16x8_to_f32(u[gg], f);
#pragma unroll
                    for (int c = 0; c < 8; ++c) s[c] += f[c];
                }
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(qbar + th * kHeadDim + c8 * 8);
        dst[0] = make_float4(s[0] / G, s[1] / G, s[2] / G, s[3] / G);
        dst[1] = make_float4(s[4] / G, s[5] / G, s[6] / G, s[7] / G);
    }
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0) flag(SPATTN_DEV_BAD_LEN);
        L = 0;
    }
    const int nb = (L + kBlock - 1) / kBlock;

    // 2. page ids of the middle blocks, once the length is known
    if (tj < a.bpc) {
        int page = -1;
        if (tblk < a.max_blocks && tblk < nb && (a.anchors || (tblk >= a.sink && tblk < nb - a.local))) {
            page = page_raw;
            if (page < 0 || page >= a.num_pages) {
                flag(SPATTN_DEV_BAD_PAGE);
                page = -1;
            }
        }
        pages[tj] = page;
    }
    __syncthreads();

    // 3. lane owns columns [4*lane, 4*lane+4) of every KV head's kbar row
    constexpr int HPC = HKV < 8 ? HKV : 8;      // heads per 8-value chunk
    constexpr int TPC = 8 / HPC;                // tokens per chunk
    for (int jb = warp; jb < a.bpc; jb += NW * BIF) {
        float4 kv[BIF][HKV];
        bool mid[BIF];
#pragma unroll
        for (int f = 0; f < BIF; ++f) {
            const int jj = jb + f * NW;
            const int page = jj < a.bpc ? pages[jj] : -1;
            mid[f] = page >= 0;
            if (mid[f]) load_kbar<HKV, KB16>(a.kbar, page, lane, kv[f]);
        }
#pragma unroll
        for (int f = 0; f < BIF; ++f) {
            const int jj = jb + f * NW;
            if (jj >= a.bpc) break;
            if (!mid[f]) {
                for (int r = lane; r < rows; r += 32) tile[r * a.bpc + jj] = -INFINITY;
                continue;
            }
            for (int t0 = 0; t0 < ntok; t0 += TPC) {
#pragma unroll
                for (int h0 = 0; h0 < HKV; h0 += HPC) {
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int tt = t0 + i / HPC, hh = h0 + i % HPC;
                        float s = 0.f;
                        if (tt < ntok) {
                            const float4 qv =
                                reinterpret_cast<const float4 *>(qbar + (tt * HKV + hh) * kHeadDim)[lane];
                            s = qv.x * kv[f][hh].x;
                            s = fmaf(qv.y, kv[f][hh].y, s);
                            s = fmaf(qv.z, kv[f][hh].z, s);
                            s = fmaf(qv.w, kv[f][hh].w, s);
                        }
                        v[i] = s;
                    }
                    const float r = reduce_scatter8(v);
                    if ((lane & 3) == 0) {
                        const int i = lane >> 2;
                        const int tt = t0 + i / HPC, hh = h0 + i % HPC;
                        if (tt < ntok) tile[(tt * HKV + hh) * a.bpc + jj] = r * a.scale;
                    }
                }
            }
        }
    }
    __syncthreads();

    // 4. coalesced store of the tile
    for (int idx = threadIdx.x; idx < rows * a.bpc; idx += kScoreThreads) {
        const int jj = idx % a.bpc, r = idx / a.bpc;
        const int j = j0 + jj;
        if (j < a.max_blocks) {
            const int hh = r % HKV, t = r / HKV;
            a.scores[(((int64_t)b * a.tq + tb + t) * HKV + hh) * a.max_blocks + j] = tile[idx];
        }
    }
}

}  // namespace spattn
