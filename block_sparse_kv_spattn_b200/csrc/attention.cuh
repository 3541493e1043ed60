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
// range is a "segment"; the CTA writes one partial (running max, sum, and
// unnormalised output per query row) per segment into slot c + unit, which
// is unique along the monotone (c, unit) staircase.  merge_kernel combines
// the partials of a unit by their log-sum-exp.
//
// Inside a CTA a producer warp walks its range and moves whole (page, head)
// K and V tiles with bulk async copies into a 3-stage shared-memory ring,
// with per-stage metadata (block id, page, unit, segment boundaries); eight
// consumer warps do QK, online softmax and PV on CUDA cores, fp32 accumulate.
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
    float *part_ml;             // [C + units][rows][2]  (max in log2 units, sum)
    int tq, hq, hkv, group, rows, units, num_pages, max_blocks, max_sel;
    float qscale;               // sm_scale * log2(e)
};

struct StageMeta {
    int j;       // logical block id
    int page;    // page id, -1 when the block or its page is invalid
    int unit;    // b * Hkv + h
    int flags;   // kFirst | kLast | kEnd
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

__host__ __device__ constexpr int attn_tile_bytes(bool fp8) { return kBlock * kHeadDim * (fp8 ? 1 : 2); }

// ring | meta | barriers | combine buffers (m per warp/row, o and l per row)
__host__ __device__ constexpr int attn_ring_bytes(bool fp8) { return kStages * 2 * attn_tile_bytes(fp8); }
__host__ __device__ constexpr int attn_smem_bytes(bool fp8, int rg) {
    return attn_ring_bytes(fp8) + kStages * 16 + (2 * kStages + 1) * 8 + kConsWarps * 4 * 4 +
           (rg < 8 ? rg * 4 * (kHeadDim + 1) * 4 : 0);
}

// Sum of v[0..15] over the 16 lanes of a half-warp, scattered: afterwards
// lane (l & 15) holds the full sum of element (l & 15).  Butterfly halving at
// offsets 8, 4, 2, 1: 15 shuffles for 16 sums.
__device__ __forceinline__ float reduce_scatter16(float (&v)[16]) {
    const int li = threadIdx.x & 15;
#pragma unroll
    for (int step = 0; step < 4; ++step) {
        const int off = 8 >> step;
        const bool up = li & off;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = up ? v[i] : v[i + off];
            const float keep = up ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

template <bool FP8>
__device__ __forceinline__ void load8(const uint8_t *tile, int tok, int li, float (&f)[8]) {
    if (FP8) {
        const uint2 u = *reinterpret_cast<const uint2 *>(tile + tok * kHeadDim + li * 8);
        e4m3x8_to_f32(u, f);
    } else {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + 2 * (tok * kHeadDim + li * 8));
        bf16x8_to_f32(u, f);
    }
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

// Count of unit u's kept list, clamped to the output capacity.
__device__ __forceinline__ int unit_count(const AttnArgs &a, int u) {
    return min(max(a.sel_count[u], 0), a.max_sel);
}

// First CTA whose range [c*W/C, (c+1)*W/C) holds flattened index x.
__host__ __device__ __forceinline__ int cta_of(int64_t x, int64_t W, int C) {
    return (int)(((x + 1) * C + W - 1) / W) - 1;
}

// RG = row groups of 4 query rows (rows = Tq * G, padded to 4 * RG).
// Consumer warp w owns RGW row groups and a slice of TPW tokens of every
// block; lanes 0-15 and 16-31 (half-warps) each take 4 tokens per 8-token
// pass, lane (l & 15) owning head-dim columns [8*(l & 15), +8).
template <int RG, bool FP8>
__global__ void __launch_bounds__(kAttnThreads, RG > 8 ? 1 : 2) attn_kernel(AttnArgs a) {
    constexpr int TILE = attn_tile_bytes(FP8);
    constexpr int RGW = RG > 8 ? RG / 8 : 1;
    constexpr int WPR = RG >= 8 ? 1 : 8 / RG;
    constexpr int TPW = kBlock / WPR;
    constexpr int NP = TPW / 8;

    extern __shared__ __align__(1024) uint8_t smem[];
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + attn_ring_bytes(FP8));
    uint64_t *full = reinterpret_cast<uint64_t *>(meta + kStages);
    uint64_t *empty = full + kStages;
    uint64_t *cbar = empty + kStages;                            // consumer barrier
    float *mbuf = reinterpret_cast<float *>(cbar + 1);           // [8 warps][4]
    float *obuf = mbuf + kConsWarps * 4;                         // [RG][4][D] (RG < 8)
    float *lbuf = obuf + RG * 4 * kHeadDim;                      // [RG][4]

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
        // total W and this CTA's range
        int64_t W = 0;
        for (int u0 = 0; u0 < a.units; u0 += 32) {
            const int u = u0 + lane;
            W += (u < a.units) ? unit_count(a, u) : 0;
        }
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        const int64_t lo = W * c / C, hi = W * (c + 1) / C;
        int i_push = 0;  // blocks pushed into the ring so far
        auto push = [&](int unit, int j, int flags) {
            const int s = i_push % kStages;
            if (i_push >= kStages && !mbar_wait(&empty[s], ((i_push / kStages) - 1) & 1)) return false;
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
            meta[s] = StageMeta{j, page, unit, flags};
            if (page >= 0) {
                const int64_t off = ((int64_t)page * a.hkv + (unit % a.hkv)) * TILE;
                uint8_t *dst = smem + s * 2 * TILE;
                mbar_arrive_expect_tx(&full[s], 2 * TILE);
                bulk_g2s(dst, a.k_cache + off, TILE, &full[s]);
                bulk_g2s(dst + TILE, a.v_cache + off, TILE, &full[s]);
            } else {
                mbar_arrive(&full[s]);
            }
            ++i_push;
            return true;
        };
        bool ok = true;
        int64_t base = 0;
        for (int u0 = 0; u0 < a.units && base < hi && ok; u0 += 32) {
            const int u = u0 + lane;
            const int cnt = (u < a.units) ? unit_count(a, u) : 0;
            int incl = warp_incl_scan(cnt);
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
                if (lane == 0) {
                    const int32_t *sel = a.sel_idx + (int64_t)unit * a.max_sel;
                    for (int i = ia; i < ib && ok; ++i)
                        ok = push(unit, sel[i], (i == ia ? kFirst : 0) | (i == ib - 1 ? kLast : 0));
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            if (ok) push(0, 0, kEnd);
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

    float qf[RGW][4][8];
    int qpos[RGW];
    float m_run[RGW], l_run[RGW], acc[RGW][4][8];
    int L = 0, unit = -1;
    uint32_t cphase = 0;

    for (int i = 0;; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1)) return;
        const StageMeta md = meta[s];
        if (md.flags & kEnd) return;
        if (md.flags & kFirst) {
            unit = md.unit;
            const int b = unit / a.hkv, h = unit % a.hkv;
            L = a.seq_lens[b];
            L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
#pragma unroll
            for (int rgi = 0; rgi < RGW; ++rgi) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int row = (rgb + rgi) * 4 + r;
                    if (row < a.rows) {
                        const int t = row / a.group, g = row % a.group;
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            a.q + (((int64_t)b * a.tq + t) * a.hq + h * a.group + g) * kHeadDim + li * 8);
                        float f[8];
                        bf16x8_to_f32(u, f);
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) qf[rgi][r][cc] = f[cc] * a.qscale;
                    } else {
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) qf[rgi][r][cc] = 0.f;
                    }
                }
                const int rowm = (rgb + rgi) * 4 + (li & 3);
                qpos[rgi] = rowm < a.rows ? L - a.tq + rowm / a.group : -1;
                m_run[rgi] = -INFINITY;
                l_run[rgi] = 0.f;
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) acc[rgi][r][cc] = 0.f;
            }
        }
        if (md.page >= 0) {
            const uint8_t *Ks = smem + s * 2 * TILE;
            const uint8_t *Vs = Ks + TILE;
            const int h = unit % a.hkv;
            const float ksc = FP8 ? a.k_scale[(int64_t)md.page * a.hkv + h] : 1.f;
            const float vsc = FP8 ? a.v_scale[(int64_t)md.page * a.hkv + h] : 1.f;
            const int base = md.j * kBlock;
            const bool need_mask = base + kBlock > L - a.tq + 1;
#pragma unroll
            for (int rgi = 0; rgi < RGW; ++rgi) {
                float sc[NP];
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    float v[16];
#pragma unroll
                    for (int tk = 0; tk < 4; ++tk) {
                        float kf[8];
                        load8<FP8>(Ks, tok0 + p * 8 + hw * 4 + tk, li, kf);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            float d = qf[rgi][r][0] * kf[0];
#pragma unroll
                            for (int cc = 1; cc < 8; ++cc) d = fmaf(qf[rgi][r][cc], kf[cc], d);
                            v[tk * 4 + r] = d;
                        }
                    }
                    float sv = reduce_scatter16(v) * ksc;
                    if (need_mask) {
                        const int pos = base + tok0 + p * 8 + hw * 4 + (li >> 2);
                        if (!(pos < L && pos <= qpos[rgi])) sv = -INFINITY;
                    }
                    sc[p] = sv;
                }
                float mx = sc[0];
#pragma unroll
                for (int p = 1; p < NP; ++p) mx = fmaxf(mx, sc[p]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[rgi], mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = exp2f(m_run[rgi] - m_use);
                m_run[rgi] = m_new;
                float pv[NP], psum = 0.f;
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    pv[p] = exp2f(sc[p] - m_use);
                    psum += pv[p];
                }
                l_run[rgi] = l_run[rgi] * alpha + psum;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float ar = __shfl_sync(0xffffffffu, alpha, r);
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) acc[rgi][r][cc] *= ar;
                }
                if (FP8) {
#pragma unroll
                    for (int p = 0; p < NP; ++p) pv[p] *= vsc;
                }
#pragma unroll
                for (int p = 0; p < NP; ++p) {
#pragma unroll
                    for (int tk = 0; tk < 4; ++tk) {
                        const int tok = tok0 + p * 8 + hw * 4 + tk;
                        float vf[8];
                        load8<FP8>(Vs, tok, li, vf);
                        if (need_mask && base + tok >= L) {
#pragma unroll
                            for (int cc = 0; cc < 8; ++cc) vf[cc] = 0.f;  // unfilled slot
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float pr = __shfl_sync(0xffffffffu, pv[p], (lane & 16) | (tk * 4 + r));
#pragma unroll
                            for (int cc = 0; cc < 8; ++cc) acc[rgi][r][cc] = fmaf(pr, vf[cc], acc[rgi][r][cc]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (md.flags & kLast) {
            // ---- end of segment: fold and write the partial to slot c + unit
            const int64_t slot = (int64_t)c + unit;
#pragma unroll
            for (int rgi = 0; rgi < RGW; ++rgi) {
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        acc[rgi][r][cc] += __shfl_xor_sync(0xffffffffu, acc[rgi][r][cc], 16);
                float l = l_run[rgi];
                l += __shfl_xor_sync(0xffffffffu, l, 4);
                l += __shfl_xor_sync(0xffffffffu, l, 8);
                l += __shfl_xor_sync(0xffffffffu, l, 16);
                l_run[rgi] = l;
            }
            if (RG >= 8) {
                // each warp owns whole rows: write directly
#pragma unroll
                for (int rgi = 0; rgi < RGW; ++rgi) {
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = (rgb + rgi) * 4 + r;
                        if (row < a.rows && lane < 16) {
                            float4 *dst = reinterpret_cast<float4 *>(
                                a.part_o + (slot * a.rows + row) * kHeadDim + li * 8);
                            dst[0] = make_float4(acc[rgi][r][0], acc[rgi][r][1], acc[rgi][r][2], acc[rgi][r][3]);
                            dst[1] = make_float4(acc[rgi][r][4], acc[rgi][r][5], acc[rgi][r][6], acc[rgi][r][7]);
                        }
                    }
                    const int rowm = (rgb + rgi) * 4 + lane;
                    if (lane < 4 && rowm < a.rows) {
                        a.part_ml[(slot * a.rows + rowm) * 2 + 0] = m_run[rgi];
                        a.part_ml[(slot * a.rows + rowm) * 2 + 1] = l_run[rgi];
                    }
                }
            } else {
                // WPR warps share each row group: combine through shared memory
                if (lane < 4) mbuf[warp * 4 + lane] = m_run[0];
                if (!consumer_sync(cbar, cphase)) return;
                float Mr[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float M = -INFINITY;
                    for (int w = rgb * WPR; w < rgb * WPR + WPR; ++w) M = fmaxf(M, mbuf[w * 4 + r]);
                    Mr[r] = M;
                }
                float f[4];
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    f[r] = Mr[r] == -INFINITY ? 0.f : exp2f(mbuf[warp * 4 + r] - Mr[r]);
                if (lane < 16) {
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            atomicAdd(&obuf[(rgb * 4 + r) * kHeadDim + li * 8 + cc], acc[0][r][cc] * f[r]);
                }
                if (lane < 4) {
                    float M = -INFINITY;
                    for (int w = rgb * WPR; w < rgb * WPR + WPR; ++w) M = fmaxf(M, mbuf[w * 4 + lane]);
                    const float fl = M == -INFINITY ? 0.f : exp2f(mbuf[warp * 4 + lane] - M);
                    atomicAdd(&lbuf[rgb * 4 + lane], l_run[0] * fl);
                }
                if (!consumer_sync(cbar, cphase)) return;
                for (int idx = threadIdx.x; idx < a.rows * kHeadDim; idx += kConsWarps * 32) {
                    const int row = idx / kHeadDim, cc = idx % kHeadDim;
                    a.part_o[(slot * a.rows + row) * kHeadDim + cc] = obuf[idx];
                    obuf[idx] = 0.f;
                    if (cc == 0) {
                        const int rg = row >> 2, r = row & 3;
                        float M = -INFINITY;
                        for (int w = rg * WPR; w < rg * WPR + WPR; ++w) M = fmaxf(M, mbuf[w * 4 + r]);
                        a.part_ml[(slot * a.rows + row) * 2 + 0] = M;
                        a.part_ml[(slot * a.rows + row) * 2 + 1] = lbuf[row];
                        lbuf[row] = 0.f;
                    }
                }
                if (!consumer_sync(cbar, cphase)) return;
            }
        }
    }
}

struct MergeArgs {
    const float *part_o;
    const float *part_ml;
    const int32_t *sel_count;
    float *out;                 // [B][Tq][Hq][D]
    int batch, tq, hq, hkv, group, rows, units, max_sel, ctas;
};

constexpr int kMergeThreads = 256;

// One warp per output row (b, t, query head): out = sum_s 2^(m_s - M) o_s /
// sum_s 2^(m_s - M) l_s over the segments of the row's unit, i.e. the slots
// c + unit for the CTAs c whose range meets the unit's part of the sequence.
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(MergeArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t grow = (int64_t)blockIdx.x * (kMergeThreads / 32) + warp;
    if (grow >= (int64_t)a.batch * a.tq * a.hq) return;
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
    float lsum = 0.f;
    if (cnt > 0) {
        // CTAs with an empty range (only when W < C) wrote no partial: skip them
        const int c_lo = cta_of(pre, W, a.ctas), c_hi = cta_of(pre + cnt - 1, W, a.ctas);
        auto nonempty = [&](int cc) { return W * (cc + 1) / a.ctas > W * cc / a.ctas; };
        float M = -INFINITY;
        for (int cc = c_lo + lane; cc <= c_hi; cc += 32)
            if (nonempty(cc)) M = fmaxf(M, a.part_ml[(((int64_t)cc + unit) * a.rows + row) * 2]);
        M = warp_max(M);
        if (M != -INFINITY) {
            for (int cc = c_lo; cc <= c_hi; ++cc) {
                if (!nonempty(cc)) continue;
                const int64_t slot = (int64_t)cc + unit;
                const float ms = a.part_ml[(slot * a.rows + row) * 2];
                const float ls = a.part_ml[(slot * a.rows + row) * 2 + 1];
                const float w = exp2f(ms - M);
                const float4 o =
                    reinterpret_cast<const float4 *>(a.part_o + (slot * a.rows + row) * kHeadDim)[lane];
                lsum = fmaf(w, ls, lsum);
                acc.x = fmaf(w, o.x, acc.x);
                acc.y = fmaf(w, o.y, acc.y);
                acc.z = fmaf(w, o.z, acc.z);
                acc.w = fmaf(w, o.w, acc.w);
            }
        }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    reinterpret_cast<float4 *>(a.out + grow * kHeadDim)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace spattn
