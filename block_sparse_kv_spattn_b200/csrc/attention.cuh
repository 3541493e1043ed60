// attention.cuh -- exact softmax attention over the kept blocks.
//
// "CSA + HCA 混合注意力机制" §2.1 / §4.4 step 4: softmax(q K_sel^T / sqrt(d)) V_sel
// over the selected entries only; §4.3: the window blocks and the partly
// filled tail block join the same softmax.  §2.3: the decode step is bound by
// reading K and V from HBM, so this kernel is a streaming reader.
//
// Work split (balanced, persistent): the kept lists of all (request, KV head)
// units are concatenated into one sequence of W blocks and CTA c of C takes
// blocks [c*W/C, (c+1)*W/C).  Each maximal run of one unit inside a CTA's
// range is a "segment"; the CTA writes one partial (running max in log2
// units, sum, unnormalised output per query row) per segment into slot
// c + unit, which is unique along the monotone (c, unit) staircase.
// merge_kernel combines the partials of a unit by their log-sum-exp.
//
// Inside a CTA a producer warp walks its range, writes each segment's query
// rows (scaled) into one of three query slots and moves whole (page, head)
// K and V tiles with bulk async copies into a 3-stage shared-memory ring,
// with per-stage metadata; eight consumer warps split each block's 64 tokens
// and do QK, online softmax and PV on CUDA cores with packed fp32 FMA.
#pragma once

#include "common.cuh"

namespace spattn {

constexpr int kConsWarps = 8;
constexpr int kAttnThreads = (kConsWarps + 1) * 32;
constexpr int kStages = 3;

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
    float *part_o;              // [C + units][rows][D]
    float *part_ml;             // [C + units][rows][2]
    int tq, hq, hkv, group, rows, units, num_pages, max_blocks, max_sel;
    float qscale;               // sm_scale * log2(e)
};

struct StageMeta {
    int j;        // logical block id
    int page;     // page id, -1 when the block or its page is invalid
    int unit;     // b * Hkv + h
    int flags;    // kFirst | kLast | kEnd
    int seg;      // segment id within the CTA (tensor-core kernel)
    int unused1;
    int qslot;    // query slot holding the segment's query rows
    int pad;
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

__host__ __device__ constexpr int attn_tile_bytes(bool fp8) { return kBlock * kHeadDim * (fp8 ? 1 : 2); }
__host__ __device__ constexpr int attn_rgw(int rg) { return rg > 8 ? rg / 8 : 1; }
__host__ __device__ constexpr int attn_tpw(int rg) { return rg >= 8 ? kBlock : kBlock / (8 / rg); }
// CTAs per SM: two while the ring and the query slots leave room for two.
__host__ __device__ constexpr int attn_ctas_per_sm(int rg) { return rg <= 2 ? 2 : 1; }

// Shared-memory layout, every region 16-byte aligned:
// ring | query slots | meta | full, empty, consumer barriers | W |
// probability buffers | segment combine (m per warp, o and l per row)
__host__ __device__ constexpr int align16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ constexpr int attn_ring_bytes(bool fp8) { return kStages * 2 * attn_tile_bytes(fp8); }
__host__ __device__ constexpr int attn_qslot_floats(int rg) { return rg * 4 * kHeadDim; }
__host__ __device__ constexpr int attn_off_qslots(bool fp8) { return attn_ring_bytes(fp8); }
__host__ __device__ constexpr int attn_off_meta(bool fp8, int rg) {
    return align16(attn_off_qslots(fp8) + kStages * attn_qslot_floats(rg) * 4);
}
__host__ __device__ constexpr int attn_off_bars(bool fp8, int rg) {
    return align16(attn_off_meta(fp8, rg) + kStages * (int)sizeof(StageMeta));
}
__host__ __device__ constexpr int attn_off_pbuf(bool fp8, int rg) {
    return align16(attn_off_bars(fp8, rg) + (2 * kStages + 1) * 8 + 16);
}
__host__ __device__ constexpr int attn_off_mbuf(bool fp8, int rg) {
    return align16(attn_off_pbuf(fp8, rg) + kConsWarps * attn_rgw(rg) * attn_tpw(rg) * 4 * 4);
}
__host__ __device__ constexpr int attn_off_obuf(bool fp8, int rg) {
    return align16(attn_off_mbuf(fp8, rg) + kConsWarps * 4 * 4);
}
__host__ __device__ constexpr int attn_smem_bytes(bool fp8, int rg) {
    return align16(attn_off_obuf(fp8, rg) + (rg < 8 ? rg * 4 * (kHeadDim + 1) * 4 : 0));
}

// Query slot layout: per row, the first halves (4 floats) of every lane's 8
// columns, then the second halves, so that 16 lanes read 16 consecutive
// float4 (no bank conflicts).
__device__ __forceinline__ int qslot_index(int row, int col) {
    const int li = col >> 3, k = col & 7;
    return row * kHeadDim + (k >> 2) * 64 + li * 4 + (k & 3);
}

// Sum of v[0..7] over the 16 lanes of a half-warp, scattered: afterwards
// lanes l and l ^ 1 hold the full sum of element ((l & 15) >> 1).  Butterfly
// halving at offsets 8, 4, 2 (each lane keeps the half named by its offset
// bit), then one xor reduction at 1: 8 shuffles for 8 sums.
__device__ __forceinline__ float reduce_scatter8_half(float (&v)[8]) {
    const int li = threadIdx.x & 15;
#pragma unroll
    for (int step = 0; step < 3; ++step) {
        const int off = 8 >> step, half = 4 >> step;
        const bool up = li & off;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// 8 consecutive head-dim values of token `tok` as 4 fp32 pairs.
template <bool FP8>
__device__ __forceinline__ void load8(const uint8_t *tile, int tok, int li, float2 (&f)[4]) {
    float x[8];
    if (FP8) {
        const uint2 u = *reinterpret_cast<const uint2 *>(tile + tok * kHeadDim + li * 8);
        e4m3x8_to_f32(u, x);
    } else {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + 2 * (tok * kHeadDim + li * 8));
        bf16x8_to_f32(u, x);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(x[2 * i], x[2 * i + 1]);
}

__device__ __forceinline__ int unit_count(const AttnArgs &a, int u) {
    return min(max(a.sel_count[u], 0), a.max_sel);
}

// CTA whose range [c*W/C, (c+1)*W/C) holds flattened index x (0 <= x < W).
__host__ __device__ __forceinline__ int cta_of(int64_t x, int64_t W, int C) {
    return (int)(((x + 1) * C + W - 1) / W) - 1;
}
__device__ __forceinline__ bool cta_nonempty(int c, int64_t W, int C) {
    return W * (c + 1) / C > W * c / C;
}

// Bounded barrier among the consumer warps: an mbarrier with one arrival per
// warp.  Returns false (status bit set by mbar_wait) if it gave up, so no
// warp can be left waiting on a warp that has already quit.
__device__ __forceinline__ bool consumer_sync(uint64_t *bar, uint32_t &phase) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase & 1);
    ++phase;
    __syncwarp();
    return ok;
}

// RG = row groups of 4 query rows (rows = Tq * G, padded to 4 * RG).
// Consumer warp w owns RGW row groups and a slice of TPW tokens of every
// block; lanes 0-15 and 16-31 (half-warps) each take 2 tokens per 4-token
// pass, lane (l & 15) owning head-dim columns [8*(l & 15), +8).
template <int RG, bool FP8>
__global__ void __launch_bounds__(kAttnThreads, attn_ctas_per_sm(RG)) attn_kernel(AttnArgs a) {
    constexpr int TILE = attn_tile_bytes(FP8);
    constexpr int RGW = attn_rgw(RG);
    constexpr int WPR = RG >= 8 ? 1 : 8 / RG;
    constexpr int TPW = attn_tpw(RG);
    constexpr int NP = TPW / 4;

    extern __shared__ __align__(1024) uint8_t smem[];
    float *qslots = reinterpret_cast<float *>(smem + attn_off_qslots(FP8));          // [kStages][RG*4][D]
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + attn_off_meta(FP8, RG));  // [kStages]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + attn_off_bars(FP8, RG));    // [kStages]
    uint64_t *empty = full + kStages;                                                  // [kStages]
    uint64_t *cbar = empty + kStages;                                                  // consumer barrier
    float *pbuf = reinterpret_cast<float *>(smem + attn_off_pbuf(FP8, RG));  // [8][RGW][TPW * 4]
    float *mbuf = reinterpret_cast<float *>(smem + attn_off_mbuf(FP8, RG));  // [8 warps][4]
    float *obuf = reinterpret_cast<float *>(smem + attn_off_obuf(FP8, RG));  // [RG][4][D] (RG < 8)
    float *lbuf = obuf + RG * 4 * kHeadDim;                                    // [RG][4]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsWarps);
        }
        mbar_init(cbar, kConsWarps);
        fence_mbar_init();
    }
    if (RG < 8)
        for (int i = threadIdx.x; i < RG * 4 * (kHeadDim + 1); i += kAttnThreads) obuf[i] = 0.f;
    __syncthreads();

    if (warp == kConsWarps) {
        // ============================================================ producer
        int64_t W = 0;
        for (int u0 = 0; u0 < a.units; u0 += 32) {
            const int u = u0 + lane;
            W += (u < a.units) ? unit_count(a, u) : 0;
        }
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        const int64_t lo = W * c / C, hi = W * (c + 1) / C;
        int i_push = 0;  // stages pushed into the ring so far
        int seg = 0;     // segments started so far
        int qs = 0;      // query slot of the current segment
        // Push one stage (called by the whole warp, uniformly).  At a segment
        // start the warp first writes the unit's query rows, scaled, into
        // query slot seg % kStages: once the stage itself is free, the
        // segment that last used that slot has been fully consumed.
        auto push = [&](int unit, int j, int flags) -> bool {
            const int s = i_push % kStages;
            int okw = 1;
            if (lane == 0 && i_push >= kStages) okw = mbar_wait(&empty[s], ((i_push / kStages) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
            if (flags & kFirst) {
                qs = seg % kStages;
                const int b = unit / a.hkv, h = unit % a.hkv;
                float *qd = qslots + qs * attn_qslot_floats(RG);
                for (int task = lane; task < RG * 4 * (kHeadDim / 8); task += 32) {
                    const int row = task / (kHeadDim / 8), c8 = task % (kHeadDim / 8);
                    float f[8];
                    if (row < a.rows) {
                        const int t = row / a.group, g = row % a.group;
                        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(
                                          a.q + (((int64_t)b * a.tq + t) * a.hq + h * a.group + g) * kHeadDim +
                                          c8 * 8),
                                      f);
                    } else {
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) f[cc] = 0.f;
                    }
                    *reinterpret_cast<float4 *>(qd + qslot_index(row, c8 * 8)) =
                        make_float4(f[0] * a.qscale, f[1] * a.qscale, f[2] * a.qscale, f[3] * a.qscale);
                    *reinterpret_cast<float4 *>(qd + qslot_index(row, c8 * 8 + 4)) =
                        make_float4(f[4] * a.qscale, f[5] * a.qscale, f[6] * a.qscale, f[7] * a.qscale);
                }
                ++seg;
            }
            __syncwarp();
            if (lane == 0) {
                int page = -1;
                if (!(flags & kEnd)) {
                    const int b = unit / a.hkv;
                    int L = a.seq_lens[b];
                    L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
                    const int nb = (L + kBlock - 1) / kBlock;
                    if (j >= 0 && j < nb) {
                        const int p = a.block_table[(int64_t)b * a.max_blocks + j];
                        if (p >= 0 && p < a.num_pages)
                            page = p;
                        else
                            flag(SPATTN_DEV_BAD_PAGE);
                    } else {
                        flag(SPATTN_DEV_BAD_BLOCK);
                    }
                }
                meta[s] = StageMeta{j, page, unit, flags, 0, 0, qs, 0};
                if (page >= 0) {
                    const int64_t off = ((int64_t)page * a.hkv + (unit % a.hkv)) * TILE;
                    uint8_t *dst = smem + s * 2 * TILE;
                    mbar_arrive_expect_tx(&full[s], 2 * TILE);
                    bulk_g2s(dst, a.k_cache + off, TILE, &full[s]);
                    bulk_g2s(dst + TILE, a.v_cache + off, TILE, &full[s]);
                } else {
                    mbar_arrive(&full[s]);
                }
            }
            ++i_push;
            return true;
        };
        bool ok = true;
        int64_t base = 0;
        for (int u0 = 0; u0 < a.units && base < hi && ok; u0 += 32) {
            const int u = u0 + lane;
            const int cnt = (u < a.units) ? unit_count(a, u) : 0;
            const int incl = warp_incl_scan(cnt);
            const int64_t ustart = base + incl - cnt;
            const bool overlap = cnt > 0 && ustart < hi && ustart + cnt > lo;
            unsigned mask = __ballot_sync(0xffffffffu, overlap);
            while (mask && ok) {
                const int src = __ffs(mask) - 1;
                mask &= mask - 1;
                const int64_t us = __shfl_sync(0xffffffffu, ustart, src);
                const int uc = __shfl_sync(0xffffffffu, cnt, src);
                const int unit = u0 + src;
                const int ia = (int)(lo > us ? lo - us : 0);
                const int ib = (int)(hi - us < uc ? hi - us : uc);
                const int32_t *sel = a.sel_idx + (int64_t)unit * a.max_sel;
                for (int i = ia; i < ib && ok; ++i)
                    ok = push(unit, sel[i], (i == ia ? kFirst : 0) | (i == ib - 1 ? kLast : 0));
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (ok) push(0, 0, kEnd);
        if (lane == 0) {
            // drain: every issued copy has landed before the CTA may exit
            for (int i = max(0, i_push - kStages); i < i_push; ++i)
                mbar_wait(&full[i % kStages], (i / kStages) & 1);
        }
        return;
    }

    // ================================================================ consumers
    const int hw = lane >> 4, li = lane & 15;
    const int rgb = RG > 8 ? warp * RGW : warp / WPR;
    const int tok0 = RG >= 8 ? 0 : (warp % WPR) * TPW;
    float *pw = pbuf + warp * RGW * TPW * 4;
    // the score this lane holds after a pass: token my_tk of the pass, row my_r
    const int my_tk = hw * 2 + (li >> 3), my_r = (li >> 1) & 3;
    uint32_t cphase = 0;

    int i = 0;  // stages consumed
    for (;;) {  // one segment per iteration
        int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1)) return;
        StageMeta md = meta[s];
        if (md.flags & kEnd) return;
        const int unit = md.unit;
        const int b = unit / a.hkv, h = unit % a.hkv;
        int L = a.seq_lens[b];
        L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
        const float *qrow = qslots + md.qslot * attn_qslot_floats(RG);

        float2 acc[RGW][4][4];
        float m_run[RGW], l_run[RGW];
        int qpos[RGW];
#pragma unroll
        for (int rgi = 0; rgi < RGW; ++rgi) {
            const int rowm = (rgb + rgi) * 4 + my_r;
            qpos[rgi] = rowm < a.rows ? L - a.tq + rowm / a.group : -1;
            m_run[rgi] = -INFINITY;
            l_run[rgi] = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) acc[rgi][r][cc] = make_float2(0.f, 0.f);
        }

        for (;;) {  // the blocks of this segment
            if (md.page >= 0) {
                const uint8_t *Ks = smem + s * 2 * TILE;
                const uint8_t *Vs = Ks + TILE;
                const float ksc = FP8 ? a.k_scale[(int64_t)md.page * a.hkv + h] : 1.f;
                const float vsc = FP8 ? a.v_scale[(int64_t)md.page * a.hkv + h] : 1.f;
                const int base = md.j * kBlock;
                const bool need_mask = base + kBlock > L - a.tq + 1;
#pragma unroll
                for (int rgi = 0; rgi < RGW; ++rgi) {
                    float sc[NP];
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        float v[8];
                        float2 k2[2][4];
                        load8<FP8>(Ks, tok0 + p * 4 + hw * 2, li, k2[0]);
                        load8<FP8>(Ks, tok0 + p * 4 + hw * 2 + 1, li, k2[1]);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float *qr = qrow + ((rgb + rgi) * 4 + r) * kHeadDim + li * 4;
                            const float4 qa = *reinterpret_cast<const float4 *>(qr);
                            const float4 qb = *reinterpret_cast<const float4 *>(qr + 64);
                            const float2 q0 = make_float2(qa.x, qa.y), q1 = make_float2(qa.z, qa.w);
                            const float2 q2 = make_float2(qb.x, qb.y), q3 = make_float2(qb.z, qb.w);
#pragma unroll
                            for (int tk = 0; tk < 2; ++tk) {
                                float2 d = __fmul2_rn(q0, k2[tk][0]);
                                d = __ffma2_rn(q1, k2[tk][1], d);
                                d = __ffma2_rn(q2, k2[tk][2], d);
                                d = __ffma2_rn(q3, k2[tk][3], d);
                                v[tk * 4 + r] = d.x + d.y;
                            }
                        }
                        float sv = reduce_scatter8_half(v) * ksc;
                        if (need_mask) {
                            const int pos = base + tok0 + p * 4 + my_tk;
                            if (!(pos < L && pos <= qpos[rgi])) sv = -INFINITY;
                        }
                        sc[p] = sv;
                    }
                    // row max over the warp's tokens: lanes sharing my_r differ in bits 0, 3, 4
                    float mx = sc[0];
#pragma unroll
                    for (int p = 1; p < NP; ++p) mx = fmaxf(mx, sc[p]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float m_new = fmaxf(m_run[rgi], mx);
                    // rescale only when some row's running max rose
                    if (__any_sync(0xffffffffu, m_new > m_run[rgi])) {
                        const float alpha = exp2f(m_run[rgi] - (m_new == -INFINITY ? 0.f : m_new));
                        l_run[rgi] *= alpha;
                        m_run[rgi] = m_new;
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float ar = __shfl_sync(0xffffffffu, alpha, 2 * r);
                            const float2 a2 = make_float2(ar, ar);
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) acc[rgi][r][cc] = __fmul2_rn(acc[rgi][r][cc], a2);
                        }
                    }
                    const float m_use = m_run[rgi] == -INFINITY ? 0.f : m_run[rgi];
                    float *pr = pw + rgi * TPW * 4;
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const float pv = exp2f(sc[p] - m_use);
                        l_run[rgi] += pv;  // lanes l and l ^ 1 hold the same value
                        if (!(li & 1)) pr[(p * 4 + my_tk) * 4 + my_r] = FP8 ? pv * vsc : pv;
                    }
                    __syncwarp();
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
#pragma unroll
                        for (int tk = 0; tk < 2; ++tk) {
                            const int tok = tok0 + p * 4 + hw * 2 + tk;
                            float2 v2[4];
                            load8<FP8>(Vs, tok, li, v2);
                            if (need_mask && base + tok >= L) {
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc) v2[cc] = make_float2(0.f, 0.f);  // unfilled slot
                            }
                            const float4 p4 = *reinterpret_cast<const float4 *>(pr + (p * 4 + hw * 2 + tk) * 4);
                            const float prow[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const float2 pp = make_float2(prow[r], prow[r]);
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc)
                                    acc[rgi][r][cc] = __ffma2_rn(pp, v2[cc], acc[rgi][r][cc]);
                            }
                        }
                    }
                    __syncwarp();
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            ++i;
            if (md.flags & kLast) break;
            s = i % kStages;
            if (!mbar_wait(&full[s], (i / kStages) & 1)) return;
            md = meta[s];
        }

        // ---- end of segment: fold the half-warps and the lanes of each row
#pragma unroll
        for (int rgi = 0; rgi < RGW; ++rgi) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    acc[rgi][r][cc].x += __shfl_xor_sync(0xffffffffu, acc[rgi][r][cc].x, 16);
                    acc[rgi][r][cc].y += __shfl_xor_sync(0xffffffffu, acc[rgi][r][cc].y, 16);
                }
            l_run[rgi] += __shfl_xor_sync(0xffffffffu, l_run[rgi], 8);
            l_run[rgi] += __shfl_xor_sync(0xffffffffu, l_run[rgi], 16);
        }
        const int64_t pbase = ((int64_t)c + unit) * a.rows;
        if (RG >= 8) {
            // each warp owns whole rows: write them
#pragma unroll
            for (int rgi = 0; rgi < RGW; ++rgi) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int row = (rgb + rgi) * 4 + r;
                    if (row < a.rows && lane < 16) {
                        float4 *dst = reinterpret_cast<float4 *>(a.part_o + (pbase + row) * kHeadDim + li * 8);
                        dst[0] = make_float4(acc[rgi][r][0].x, acc[rgi][r][0].y, acc[rgi][r][1].x, acc[rgi][r][1].y);
                        dst[1] = make_float4(acc[rgi][r][2].x, acc[rgi][r][2].y, acc[rgi][r][3].x, acc[rgi][r][3].y);
                    }
                }
                const int rowm = (rgb + rgi) * 4 + (lane >> 1);
                if (lane < 8 && !(lane & 1) && rowm < a.rows)
                    *reinterpret_cast<float2 *>(a.part_ml + (pbase + rowm) * 2) = make_float2(m_run[rgi], l_run[rgi]);
            }
        } else {
            // WPR warps share each row group: combine through shared memory
            if (lane < 8 && !(lane & 1)) mbuf[warp * 4 + (lane >> 1)] = m_run[0];
            if (!consumer_sync(cbar, cphase)) return;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float M = -INFINITY;
                for (int w = rgb * WPR; w < rgb * WPR + WPR; ++w) M = fmaxf(M, mbuf[w * 4 + r]);
                const float f = M == -INFINITY ? 0.f : exp2f(mbuf[warp * 4 + r] - M);
                if (lane < 16) {
                    float *o = obuf + (rgb * 4 + r) * kHeadDim + li * 8;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        atomicAdd(o + 2 * cc, acc[0][r][cc].x * f);
                        atomicAdd(o + 2 * cc + 1, acc[0][r][cc].y * f);
                    }
                }
                if (lane == 2 * r) atomicAdd(&lbuf[rgb * 4 + r], l_run[0] * f);
            }
            if (!consumer_sync(cbar, cphase)) return;
            for (int idx = threadIdx.x; idx < a.rows * kHeadDim; idx += kConsWarps * 32) {
                const int row = idx / kHeadDim, cc = idx % kHeadDim;
                a.part_o[(pbase + row) * kHeadDim + cc] = obuf[idx];
                obuf[idx] = 0.f;
                if (cc == 0) {
                    const int rg = row >> 2, r = row & 3;
                    float M = -INFINITY;
                    for (int w = rg * WPR; w < rg * WPR + WPR; ++w) M = fmaxf(M, mbuf[w * 4 + r]);
                    a.part_ml[(pbase + row) * 2 + 0] = M;
                    a.part_ml[(pbase + row) * 2 + 1] = lbuf[row];
                    lbuf[row] = 0.f;
                }
            }
            if (!consumer_sync(cbar, cphase)) return;
        }
    }
}

struct MergeArgs {
    const float *part_o;
    const float *part_ml;
    const int32_t *sel_count;
    float *out;                 // [B][Tq][Hq][D]
    float *lse;                 // nullable: [B][Tq][Hq], ln of the row's sum of exp(logit)
    int batch, tq, hq, hkv, group, rows, units, max_sel, ctas;
    int wslots;                 // partial records per (CTA, unit): 1, 2 (hi / lo parts) or 4 (per softmax warp)
    int pairs;                  // 4 records: warp w's pair w / 2 took only tiles of its parity
};

constexpr int kMergeMaxWarps = 8;   // warps per output row, for units split over many CTAs

// Record x of a unit's candidate list (CTA c_lo + x / wslots, warp x %
// wslots), or -1 if it was not written: the CTA's range misses the unit's
// [pre, pre + cnt) part (only when W < C), or, with one record per
// tensor-core softmax warp, the warp's pair took none of the CTA's tiles of
// the unit (pair p takes CTA-local tile indices of parity p).
__device__ __forceinline__ int64_t merge_record(const MergeArgs &a, int x, int c_lo, int unit, int64_t pre, int cnt,
                                                int64_t W) {
    const int cc = c_lo + x / a.wslots, w = x % a.wslots;
    const int64_t lo_c = W * cc / a.ctas, hi_c = W * (cc + 1) / a.ctas;
    const int64_t ia = (pre > lo_c ? pre : lo_c) - lo_c;
    const int64_t ib = (pre + cnt < hi_c ? pre + cnt : hi_c) - lo_c;
    if (ib <= ia) return -1;
    if (a.pairs && ib - ia < 2 && (ia & 1) != (w >> 1)) return -1;
    return ((int64_t)cc + unit) * a.wslots + w;
}

// One CTA per output row (b, t, query head): out = sum_s 2^(m_s - M) o_s /
// sum_s 2^(m_s - M) l_s over the partial records of the row's unit: slot
// c + unit for each CTA c whose range meets the unit's part of the sequence
// (with wslots = 4, record w of that slot for each softmax warp w whose pair
// took one of the CTA's tiles of the unit: pair w / 2 takes the tiles with
// CTA-local index of its parity).  The CTA's warps take batches of 32
// records in turn (a unit split over many CTAs has hundreds) and are
// combined through shared memory.  A unit with nothing kept gets a zero row.
__global__ void __launch_bounds__(kMergeMaxWarps * 32) merge_kernel(MergeArgs a) {
    __shared__ float s_m[kMergeMaxWarps], s_l[kMergeMaxWarps];
    __shared__ float4 s_acc[kMergeMaxWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int64_t grow = blockIdx.x;
    const int i = (int)(grow % a.hq);
    const int t = (int)((grow / a.hq) % a.tq);
    const int b = (int)(grow / ((int64_t)a.hq * a.tq));
    const int h = i / a.group, g = i % a.group;
    const int unit = b * a.hkv + h;
    const int row = t * a.group + g;
    // prefix of the unit in the concatenated sequence, and the total W
    int64_t pre = 0, W = 0;
    for (int u = lane; u < a.units; u += 32) {
        const int cnt = min(max(a.sel_count[u], 0), a.max_sel);
        W += cnt;
        if (u < unit) pre += cnt;
    }
    for (int o = 16; o > 0; o >>= 1) {
        pre += __shfl_xor_sync(0xffffffffu, pre, o);
        W += __shfl_xor_sync(0xffffffffu, W, o);
    }
    const int cnt = min(max(a.sel_count[unit], 0), a.max_sel);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f, M = -INFINITY;
    if (cnt > 0) {
        // records r = (slot * wslots + w) that were written: CTAs with an
        // empty range (only when W < C) wrote none; with wslots = 4 a pair
        // wrote only if it took a tile
        const int c_lo = cta_of(pre, W, a.ctas), c_hi = cta_of(pre + cnt - 1, W, a.ctas);
        const int nrec = (c_hi - c_lo + 1) * a.wslots;
        // batches of 32 records, one per lane, merged online: the lanes load
        // their records' (m, l) together, then the row's O of every record of
        // the batch is loaded in one unrolled run (no record waits on another)
        for (int x0 = 32 * warp; x0 < nrec; x0 += 32 * nw) {
            const int64_t r = x0 + lane < nrec ? merge_record(a, x0 + lane, c_lo, unit, pre, cnt, W) : -1;
            float2 ml = make_float2(-INFINITY, 0.f);
            if (r >= 0) ml = *reinterpret_cast<const float2 *>(a.part_ml + (r * a.rows + row) * 2);
            const float Mb = fmaxf(M, warp_max(ml.x));
            const unsigned valid = __ballot_sync(0xffffffffu, r >= 0 && ml.x != -INFINITY);
            if (Mb == -INFINITY || !valid) continue;   // uniform: nothing to add
            if (Mb != M) {   // uniform: rescale what is summed so far
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
            // records without weight read the first valid one (weight 0)
            const int64_t rfirst = __shfl_sync(0xffffffffu, r, __ffs(valid) - 1);
            const int64_t rr = ((valid >> lane) & 1u) ? r : rfirst;
            const int n_here = nrec - x0 < 32 ? nrec - x0 : 32;
#pragma unroll 16
            for (int e = 0; e < n_here; ++e) {
                const float we = __shfl_sync(0xffffffffu, w, e);
                const int64_t re = __shfl_sync(0xffffffffu, rr, e);
                const float4 o = reinterpret_cast<const float4 *>(a.part_o + (re * a.rows + row) * kHeadDim)[lane];
                acc.x = fmaf(we, o.x, acc.x);
                acc.y = fmaf(we, o.y, acc.y);
                acc.z = fmaf(we, o.z, acc.z);
                acc.w = fmaf(we, o.w, acc.w);
            }
        }
        lsum = warp_sum(lsum);
    }
    if (nw > 1) {
        // combine the warps: weights 2^(M_w - M)
        if (lane == 0) {
            s_m[warp] = M;
            s_l[warp] = lsum;
        }
        s_acc[warp][lane] = acc;
        __syncthreads();
        if (warp != 0) return;
        float Mt = -INFINITY;
        for (int w = 0; w < nw; ++w) Mt = fmaxf(Mt, s_m[w]);
        M = Mt;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        lsum = 0.f;
        if (Mt != -INFINITY)
            for (int w = 0; w < nw; ++w) {
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
