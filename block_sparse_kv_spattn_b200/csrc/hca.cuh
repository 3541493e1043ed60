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

struct HcaPoolArgs {
    const uint8_t *k_cache, *v_cache;   // bf16 or e4m3 bytes [num_pages][Hkv][P][D]
    const float *k_scale, *v_scale;     // fp8 only
    const int32_t *block_table;
    const int32_t *old_lens;            // nullable: every entry
    const int32_t *seq_lens;
    float *khat, *vhat;                 // [B][Hkv][G_max][D]: a (request, KV head)'s entries contiguous
    int hkv, num_pages, max_blocks, gmax;
};

constexpr int kHcaPoolThreads = 512;

// Grid (gx, B), kHcaPoolThreads threads; the CTAs stride over the entries.
// Without old_lens every entry is written (zeros past the end of the
// request); with old_lens only the entries that hold a token of
// [old_len, L).  Per entry, half-warp j of 32 takes KV head j % Hkv and every
// (32 / Hkv)-th token from token j / Hkv, 8 columns per lane in fp32 (fp8
// codes times their page's scale); the half-warps' sums are combined in a
// fixed order through shared memory and divided by the token count.
template <bool FP8>
__global__ void __launch_bounds__(kHcaPoolThreads) hca_pool_kernel(HcaPoolArgs a) {
    __shared__ float4 s_k[32][32], s_v[32][32];   // [half-warp][16 lanes x 8 columns as 2 float4]
    __shared__ int s_page[kHcaGroupBlocks];
    const int b = blockIdx.y;
    const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
    const int h = hw % a.hkv, tl = hw / a.hkv, ntl = 32 / a.hkv;
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
        if (threadIdx.x < kHcaGroupBlocks) {
            const int j = g * kHcaGroupBlocks + threadIdx.x;
            int page = -1;
            if (t0 + (int)threadIdx.x * kBlock < t1) {
                page = a.block_table[(int64_t)b * a.max_blocks + j];
                if (page < 0 || page >= a.num_pages) {
                    flag(SPATTN_DEV_BAD_PAGE);
                    page = -1;
                }
            }
            s_page[threadIdx.x] = page;
        }
        __syncthreads();
        float k8[8], v8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) k8[c] = v8[c] = 0.f;
#pragma unroll 4
        for (int t = t0 + tl; t < t1; t += ntl) {
            const int page = s_page[(t - t0) / kBlock];
            if (page < 0) continue;
            const int64_t off = (((int64_t)page * a.hkv + h) * kBlock + (t % kBlock)) * kHeadDim + hl * 8;
            float kx[8], vx[8];
            if (FP8) {
                const float ks = a.k_scale[(int64_t)page * a.hkv + h], vs = a.v_scale[(int64_t)page * a.hkv + h];
                e4m3x8_to_f32(*reinterpret_cast<const uint2 *>(a.k_cache + off), kx);
                e4m3x8_to_f32(*reinterpret_cast<const uint2 *>(a.v_cache + off), vx);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    k8[c] = fmaf(kx[c], ks, k8[c]);
                    v8[c] = fmaf(vx[c], vs, v8[c]);
                }
            } else {
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.k_cache + off * 2), kx);
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.v_cache + off * 2), vx);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    k8[c] += kx[c];
                    v8[c] += vx[c];
                }
            }
        }
        s_k[hw][2 * hl] = make_float4(k8[0], k8[1], k8[2], k8[3]);
        s_k[hw][2 * hl + 1] = make_float4(k8[4], k8[5], k8[6], k8[7]);
        s_v[hw][2 * hl] = make_float4(v8[0], v8[1], v8[2], v8[3]);
        s_v[hw][2 * hl + 1] = make_float4(v8[4], v8[5], v8[6], v8[7]);
        __syncthreads();
        // thread -> (K or V, head, 4 columns): sum the head's half-warps in order
        const float inv = t1 > t0 ? 1.f / (float)(t1 - t0) : 0.f;
        for (int task = threadIdx.x; task < 2 * a.hkv * 32; task += kHcaPoolThreads) {
            const int kv = task / (a.hkv * 32), hh = (task / 32) % a.hkv, c4 = task % 32;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < ntl; ++j) {
                const float4 x = kv ? s_v[j * a.hkv + hh][c4] : s_k[j * a.hkv + hh][c4];
                acc.x += x.x, acc.y += x.y, acc.z += x.z, acc.w += x.w;
            }
            float *dst = kv ? a.vhat : a.khat;
            reinterpret_cast<float4 *>(dst + (((int64_t)b * a.hkv + hh) * a.gmax + g) * kHeadDim)[c4] =
                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
        __syncthreads();   // s_page and the partials are reused by the next entry
    }
}

struct HcaAttendArgs {
    const uint16_t *q;          // bf16 bits [B][Tq][Hq][D]
    const float *khat, *vhat;   // [B][Hkv][G_max][D]
    const int32_t *seq_lens;
    float *part_o;              // [units][split][rows][D]: unnormalised partial outputs
    float *part_ml;             // [units][split][rows][2]: base-2 maximum and sum
    int tq, hq, hkv, max_blocks, gmax, split;
    float qscale;               // sm_scale * log2(e)
};

constexpr int kHcaMaxSplit = 16;    // CTAs per (request, KV head), at most
constexpr int kHcaCtaWarps = 8;     // consumer warps per CTA (plus one producer warp)
constexpr int kHcaWarpsPerStage = 4;   // consumer warps sharing one stage

// Entries of request length L visible to the query token at position qpos:
// the full entries up to qpos, plus the last partial one at qpos = L - 1.
__device__ __forceinline__ int hca_visible(int L, int qpos) {
    if (qpos < 0) return 0;
    const int full = (qpos + 1) / kHcaTokens;
    return (qpos + 1 == L && L % kHcaTokens) ? full + 1 : full;
}

// Sum over the warp of 32 values per lane, scattered: lane j ends with the
// total of value j.  Five butterfly rounds; each keeps the half of the
// values its side of the exchange owns (16 + 8 + 4 + 2 + 1 shuffles).
__device__ __forceinline__ float warp_reduce_scatter32(float (&x)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool hi = lane & w;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float keep = hi ? x[i + w] : x[i];
            const float send = hi ? x[i] : x[i + w];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return x[0];
}

// Wait (bounded, ~1 s) until the producer has issued stage use `it`.
__device__ __forceinline__ bool hca_wait_issued(const int *slot, int it) {
    const volatile int *v = slot;
    if (*v == it) return true;
    const uint64_t t0 = global_ns();
    while (*v != it) {
        if (global_ns() - t0 > kWaitLimitNs) {
            flag(SPATTN_DEV_WAIT_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

// Stages of the entry ring: K and V of kHcaWarpsPerStage * E entries each;
// 96 KiB (E = 8) or 80 KiB (E = 4) in all, so that two CTAs fit on an SM.
template <int E>
struct HcaRing {
    static constexpr int kChunk = kHcaWarpsPerStage * E;       // entries per stage
    static constexpr int kStages = E == 8 ? 3 : 5;
    static constexpr int kStageBytes = 2 * kChunk * kHeadDim * 4;
    static constexpr int kSmem = kStages * kStageBytes;
};

// Grid (split, B * Hkv): CTA c of (request b, KV head h) takes share c of the
// entries visible to the last query token.  A producer warp streams the
// share's K and V means (contiguous in the [B][Hkv][G][D] layout) through a
// ring of shared-memory stages with bulk async copies.  The consumer warps
// form two teams of kHcaWarpsPerStage that take alternate stages, E entries
// per warp.  A warp holds RQ query rows of the unit (rows are (token, query
// head of the group)): the lanes hold 4 columns each, RQ x E = 32 dot
// products are reduced and scattered so that lane j owns score j (row
// j / E, entry j % E), which takes one exp2 per lane; probabilities go
// through shared memory to every lane for the P V update.  At the end of a
// pass the warps' partials go to the idle ring, are combined, and the CTA
// writes one partial record per row (maximum, sum, unnormalised output);
// hca_combine_kernel merges the records.  More than RQ rows: passes over
// the rows, each streaming the entries again.  Every wait is bounded
// (SPATTN_DEV_WAIT_TIMEOUT).
template <int RQ, int E>
__global__ void __launch_bounds__((kHcaCtaWarps + 1) * 32, RQ == 4 ? 2 : 1) hca_partial_kernel(HcaAttendArgs a) {
    static_assert(RQ * E == 32, "one score per lane");
    using R = HcaRing<E>;
    static_assert(kHcaCtaWarps * RQ * 32 * 16 + 2 * kHcaCtaWarps * RQ * 4 <= R::kSmem, "partials fit the ring");
    extern __shared__ __align__(128) unsigned char ring[];
    __shared__ __align__(8) uint64_t full[R::kStages], empty[R::kStages];
    __shared__ int s_chunk[R::kStages];   // stage use (it) whose copies were issued last
    __shared__ __align__(16) float s_p[kHcaCtaWarps][32];
    __shared__ int s_dead;
    // end-of-pass partials of the warps, over the (then idle) ring
    float4(*s_acc)[RQ][32] = reinterpret_cast<float4(*)[RQ][32]>(ring);
    float(*s_m)[RQ] = reinterpret_cast<float(*)[RQ]>(ring + kHcaCtaWarps * RQ * 32 * 16);
    float(*s_l)[RQ] = s_m + kHcaCtaWarps;
    const int crank = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.y, b = unit / a.hkv, h = unit % a.hkv;
    const int grp = a.hq / a.hkv, rows = a.tq * grp;
    int L = a.seq_lens[b];
    L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
    const int ng = hca_visible(L, L - 1);          // the last query token sees the most
    const int c_lo = (int)((int64_t)ng * crank / a.split), c_hi = (int)((int64_t)ng * (crank + 1) / a.split);
    const int nchunks = (c_hi - c_lo + R::kChunk - 1) / R::kChunk;
    const int64_t ubase = ((int64_t)unit * a.gmax + c_lo) * kHeadDim;   // first float of the share
    const int64_t rec0 = ((int64_t)unit * a.split + crank) * rows;       // this CTA's first record
    if (threadIdx.x == 0) {
        for (int s = 0; s < R::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kHcaWarpsPerStage);
            s_chunk[s] = -1;
        }
        s_dead = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int team = warp / kHcaWarpsPerStage, wslot = warp % kHcaWarpsPerStage;
    const int my_r = lane / E, my_e = lane % E;
    bool dead = false;     // a wait gave up: skip the remaining waits
    int base = 0;          // stage uses before this pass

    for (int r0 = 0; r0 < rows; r0 += RQ, base += nchunks) {
        float m[RQ], l_lane = 0.f;
        float4 acc[RQ];
#pragma unroll
        for (int r = 0; r < RQ; ++r) {
            m[r] = -INFINITY;
            acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (warp == kHcaCtaWarps) {
            // producer: stream the share's chunks of K and V
            if (lane == 0)
                for (int c = 0; c < nchunks; ++c) {
                    const int it = base + c, s = it % R::kStages;
                    if (it >= R::kStages && !dead && !mbar_wait(&empty[s], ((it / R::kStages) - 1) & 1)) {
                        dead = true;
                        s_dead = 1;
                    }
                    if (dead) continue;
                    const int n = min(R::kChunk, c_hi - c_lo - c * R::kChunk);
                    const uint32_t bytes = (uint32_t)n * kHeadDim * 4;
                    unsigned char *st = ring + s * R::kStageBytes;
                    *reinterpret_cast<volatile int *>(&s_chunk[s]) = it;
                    __threadfence_block();
                    mbar_arrive_expect_tx(&full[s], 2 * bytes);
                    bulk_g2s(st, a.khat + ubase + (int64_t)c * R::kChunk * kHeadDim, bytes, &full[s]);
                    bulk_g2s(st + R::kStageBytes / 2, a.vhat + ubase + (int64_t)c * R::kChunk * kHeadDim, bytes,
                             &full[s]);
                }
        } else {
            float4 qv[RQ];
            int vis[RQ];
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                const int rr = r0 + r;
                qv[r] = make_float4(0.f, 0.f, 0.f, 0.f);
                vis[r] = 0;
                if (rr < rows) {
                    const int t = rr / grp, gi = rr % grp;
                    const uint2 qu = reinterpret_cast<const uint2 *>(
                        a.q + (((int64_t)b * a.tq + t) * a.hq + h * grp + gi) * kHeadDim)[lane];
                    qv[r] = make_float4(bf16lo(qu.x) * a.qscale, bf16hi(qu.x) * a.qscale,
                                        bf16lo(qu.y) * a.qscale, bf16hi(qu.y) * a.qscale);
                    vis[r] = hca_visible(L, L - a.tq + t);
                }
            }
            int my_vis = vis[0];
#pragma unroll
            for (int r = 1; r < RQ; ++r) my_vis = my_r == r ? vis[r] : my_vis;
            for (int c = team; c < nchunks; c += kHcaCtaWarps / kHcaWarpsPerStage) {
                const int it = base + c, s = it % R::kStages;
                // the two teams take alternate stage uses, so one team may
                // reach a stage's next use while the other still holds the
                // current one: the parity wait alone would take the phase in
                // progress for the one wanted, so first see that this use's
                // copies were issued
                if (!dead && !hca_wait_issued(&s_chunk[s], it)) {
                    dead = true;
                    s_dead = 1;
                }
                if (!dead && !mbar_wait(&full[s], (it / R::kStages) & 1)) {
                    dead = true;
                    s_dead = 1;
                }
                if (dead) continue;
                const int g = c_lo + c * R::kChunk + wslot * E;     // this warp's first entry
                const int n = min(E, c_hi - g);                      // may be <= 0 in the last chunk
                const float4 *ks =
                    reinterpret_cast<const float4 *>(ring + s * R::kStageBytes) + wslot * E * 32 + lane;
                const float4 *vs = ks + R::kChunk * 32;
                if (n > 0) {
                    float x[32];
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const float4 k = ks[(e < n ? e : 0) * 32];
#pragma unroll
                        for (int r = 0; r < RQ; ++r) {
                            float d = qv[r].x * k.x;
                            d = fmaf(qv[r].y, k.y, d);
                            d = fmaf(qv[r].z, k.z, d);
                            x[r * E + e] = fmaf(qv[r].w, k.w, d);
                        }
                    }
                    float sc = warp_reduce_scatter32(x);
                    if (my_e >= n || g + my_e >= my_vis) sc = -INFINITY;
                    // row maxima over the row's E lanes, then to every lane
                    float mb = sc;
#pragma unroll
                    for (int o = 1; o < E; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
                    float f_my = 1.f, m_my = -INFINITY;
#pragma unroll
                    for (int r = 0; r < RQ; ++r) {
                        const float mn = fmaxf(m[r], __shfl_sync(0xffffffffu, mb, r * E));
                        const float f = mn == m[r] ? 1.f : exp2f(m[r] - mn);   // uniform per row
                        acc[r].x *= f, acc[r].y *= f, acc[r].z *= f, acc[r].w *= f;
                        m[r] = mn;
                        f_my = my_r == r ? f : f_my;
                        m_my = my_r == r ? mn : m_my;
                    }
                    const float p = sc == -INFINITY ? 0.f : exp2f(sc - m_my);
                    l_lane = fmaf(l_lane, f_my, p);
                    s_p[warp][lane] = p;
                    __syncwarp();
#pragma unroll
                    for (int e4 = 0; e4 < E; e4 += 4) {
                        float4 v[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) v[j] = vs[(e4 + j < n ? e4 + j : 0) * 32];
#pragma unroll
                        for (int r = 0; r < RQ; ++r) {
                            const float4 pp = *reinterpret_cast<const float4 *>(&s_p[warp][r * E + e4]);
                            const float pe[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                acc[r].x = fmaf(pe[j], v[j].x, acc[r].x);
                                acc[r].y = fmaf(pe[j], v[j].y, acc[r].y);
                                acc[r].z = fmaf(pe[j], v[j].z, acc[r].z);
                                acc[r].w = fmaf(pe[j], v[j].w, acc[r].w);
                            }
                        }
                    }
                }
                __syncwarp();   // the stage and s_p are read
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            // the warp's rows: l summed over each row's E lanes
#pragma unroll
            for (int o = 1; o < E; o <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);
        }
        __syncthreads();   // the ring is idle: every chunk of the pass was consumed
        if (warp < kHcaCtaWarps) {
            if (my_e == 0) s_l[warp][my_r] = l_lane;
            if (lane < RQ) {
                float mm = m[0];
#pragma unroll
                for (int r = 1; r < RQ; ++r) mm = lane == r ? m[r] : mm;
                s_m[warp][lane] = mm;
            }
#pragma unroll
            for (int r = 0; r < RQ; ++r) s_acc[warp][r][lane] = acc[r];
        }
        __syncthreads();
        // the CTA's record per row (consumer warp w takes rows w, w + 8, ...)
        if (warp < kHcaCtaWarps)
            for (int r = warp; r < RQ && r0 + r < rows; r += kHcaCtaWarps) {
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kHcaCtaWarps; ++w) M = fmaxf(M, s_m[w][r]);
                float lt = 0.f;
                float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
                if (M != -INFINITY)
#pragma unroll
                    for (int w = 0; w < kHcaCtaWarps; ++w) {
                        const float f = s_m[w][r] == -INFINITY ? 0.f : exp2f(s_m[w][r] - M);
                        const float4 o = s_acc[w][r][lane];
                        lt = fmaf(f, s_l[w][r], lt);
                        at.x = fmaf(f, o.x, at.x), at.y = fmaf(f, o.y, at.y);
                        at.z = fmaf(f, o.z, at.z), at.w = fmaf(f, o.w, at.w);
                    }
                const int64_t rec = rec0 + r0 + r;
                reinterpret_cast<float4 *>(a.part_o + rec * kHeadDim)[lane] = at;
                if (lane == 0) *reinterpret_cast<float2 *>(a.part_ml + rec * 2) = make_float2(M, lt);
            }
        __syncthreads();   // the partials were read: the next pass's copies may land
    }
    // after a wait gave up, copies may still be in flight into this CTA's
    // ring: give the last stages' transfers a bounded time to land
    const int used = base;
    if (s_dead && threadIdx.x == kHcaCtaWarps * 32)
        for (int j = used > R::kStages ? used - R::kStages : 0; j < used; ++j)
            if (!mbar_wait(&full[j % R::kStages], (j / R::kStages) & 1)) break;
}

struct HcaCombineArgs {
    const float *part_o, *part_ml;   // as HcaAttendArgs
    const float *base_out;           // nullable: another branch's result to merge with
    const float *base_lse;           //   ([B][Tq][Hq][D] and [B][Tq][Hq], natural log)
    float *out;                      // [B][Tq][Hq][D]
    float *lse;                      // [B][Tq][Hq], natural log; nullable
    int64_t nrows;                   // B * Tq * Hq
    int tq, hq, hkv, split;
};

// One warp per output row (b, t, query head): the split partial records of
// the row's (request, KV head) -- lane k holds record k's (m, l) -- and, if
// given, the other branch's (out, lse) as one more term with m = lse log2(e)
// and l = 1: out = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k.
__global__ void __launch_bounds__(256) hca_combine_kernel(HcaCombineArgs a) {
    const int64_t grow = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (grow >= a.nrows) return;
    const int i = (int)(grow % a.hq), t = (int)((grow / a.hq) % a.tq), b = (int)(grow / ((int64_t)a.hq * a.tq));
    const int grp = a.hq / a.hkv, h = i / grp, rows = a.tq * grp;
    const int64_t rec0 = ((int64_t)(b * a.hkv + h) * a.split) * rows + t * grp + i % grp;
    float2 ml = make_float2(-INFINITY, 0.f);
    if (lane < a.split) ml = *reinterpret_cast<const float2 *>(a.part_ml + (rec0 + (int64_t)lane * rows) * 2);
    const float bm = a.base_out ? a.base_lse[grow] * kLog2e : -INFINITY;
    const float M = fmaxf(warp_max(ml.x), bm);
    float lt = 0.f;
    float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
        const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
        lt = warp_sum(w * ml.y);
        for (int k = 0; k < a.split; ++k) {
            const float wk = __shfl_sync(0xffffffffu, w, k);
            if (wk == 0.f) continue;   // uniform
            const float4 o = reinterpret_cast<const float4 *>(a.part_o + (rec0 + (int64_t)k * rows) * kHeadDim)[lane];
            at.x = fmaf(wk, o.x, at.x), at.y = fmaf(wk, o.y, at.y);
            at.z = fmaf(wk, o.z, at.z), at.w = fmaf(wk, o.w, at.w);
        }
        if (bm != -INFINITY) {
            const float f = exp2f(bm - M);
            const float4 o = reinterpret_cast<const float4 *>(a.base_out + grow * kHeadDim)[lane];
            lt += f;
            at.x = fmaf(f, o.x, at.x), at.y = fmaf(f, o.y, at.y);
            at.z = fmaf(f, o.z, at.z), at.w = fmaf(f, o.w, at.w);
        }
    }
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    __syncwarp();   // every lane has read the other branch's row: out / lse may be those buffers
    reinterpret_cast<float4 *>(a.out + grow * kHeadDim)[lane] =
        make_float4(at.x * inv, at.y * inv, at.z * inv, at.w * inv);
    if (a.lse && lane == 0) a.lse[grow] = lt > 0.f ? (M + log2f(lt)) * 0.69314718055994531f : -INFINITY;
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
