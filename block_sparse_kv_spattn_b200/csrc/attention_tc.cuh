// attention_tc.cuh -- exact softmax attention over the kept blocks on the
// sm_100a tensor cores (tcgen05, accumulators in TMEM), bf16 caches.
//
// "CSA + HCA 混合注意力机制" §2.1 / §4.4 step 4: softmax(q K_sel^T / sqrt(d)) V_sel
// over the selected entries only (§4.3: window and partly filled tail join).
//
// Work split, segments and query slots are those of attention.cuh: the kept
// lists of all (request, KV head) units are concatenated and cut into equal
// ranges, one per CTA of a persistent grid; a CTA's range falls into
// segments, one per unit it meets.
//
// Two pairs of softmax warps take the blocks of a CTA in turn: pair 0
// (warps 0, 1) the even ones, pair 1 (warps 2, 3) the odd ones; inside a
// pair each warp owns 32 of the block's 64 tokens.  Every softmax warp keeps
// its own reference maximum m per query row, its own row sums and its own
// output accumulator, and writes its own partial record at the end of each
// segment it took part in; merge_kernel combines the records by
// log-sum-exp.  The softmax warps therefore never wait on one another.
//
// Products, with NQ = 16 query rows of the unit (the group's heads times the
// chunk's tokens, zero padded):
//   S^T [128 x NQ]  = K [128 x d] . Q^T [d x NQ]   K-major A and B.  Rows
//                     0-63 are the tokens of an even tile (pair 0), rows
//                     64-127 those of the following odd tile (pair 1), so
//                     each warp reads its tokens from its own TMEM lane
//                     quarter.  The ring keeps each K box of consecutive
//                     stages adjacent, so one product serves both tiles when
//                     they belong to the same segment ("joint"); otherwise
//                     each tile gets its own product and the other 64 rows
//                     are whatever lies next to it (never read).  S is double
//                     buffered, so the next products run while the pairs
//                     still work on the current ones.
//   O [128 x d]    += P [128 x 64] . V [64 x d]    K-major A, MN-major B.
//                     Row 32w + r of P holds warp w's weights hi(p) of query
//                     row r, row 32w + 16 + r the remainders lo(p) = p - hi(p)
//                     (hi, lo bf16: ~16 significant bits together), nonzero
//                     only at the warp's own 32 tokens.  So O's TMEM lanes
//                     32w .. 32w + 31 are warp w's accumulator (hi and lo
//                     parts of each row, added at the end); each pair has its
//                     own O columns, so no product of one pair touches the
//                     other pair's accumulator.
//
// Reference maximum: p = 2^(x - m), m the warp's reference for the row.  m
// starts at -inf and is raised (accumulator and sums scaled by 2^(m_old -
// m_new)) only when a score exceeds it by more than kTcSlack; otherwise
// weights up to 2^kTcSlack enter the sums, well inside fp32 and bf16 range.
// The first visible block sets m and later ones rarely move it, so the
// common path has no cross-lane reduction and no accumulator traffic.
//
// Warps: 0-3 softmax (TMEM lanes 0-127), 4 producer (TMA + query slots),
// 5 MMA issue (one lane) and TMEM owner.
#pragma once

#include "attention.cuh"
#include "tcgen05.cuh"

namespace spattn {

constexpr int kTcThreads = 6 * 32;
constexpr int kTcNQ = 16;                      // query rows per product (N of S^T)
constexpr int kTcBox = 8192;                   // one 64 x 64 bf16 box
constexpr int kTcStageBytes = 4 * kTcBox;      // K box 0, K box 1, V box 0, V box 1 of a tile
constexpr int kJoint = 8;                      // StageMeta flag: S of this odd tile came with the even one
constexpr int kTcWarpSlots = 4;                // partial records per (CTA, unit)
constexpr int kTcTmemCols = 512;               // S: 4 x NQ | O: 2 x 128
constexpr float kTcSlack = 16.f;               // log2 headroom above the reference

// Shared-memory layout for RQ processed query rows.  Query slots first (a
// product with N = 16 reads rows 8-15 past a slot of 8 rows; those columns
// of S are never used, and the bytes read are the next slot or P), then P
// (128 rows x 64 bf16), the ring as four arrays of boxes [K0 | K1 | V0 |
// V1][stage] so that the K boxes of stages 2k and 2k + 1 are adjacent, the
// stage metadata and the barriers.  Even stage counts: 6 when a slot needs
// only 8 rows, else 4 (227 KiB per CTA).
template <int RQ>
struct TcLayout {
    static constexpr int kStages = RQ <= 8 ? 6 : 4;
    static constexpr int kQRows = RQ <= 8 ? 8 : 16;
    static constexpr int kQSlot = kQRows * 256;
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + kStages * kQSlot;
    static constexpr int kOffRing = kOffP + 128 * 128;
    static constexpr int kOffMeta = kOffRing + kStages * kTcStageBytes;
    static constexpr int kNBars = 2 * kStages + 12 + 2;
    static constexpr int kOffBars = align16(kOffMeta + kStages * 32);
    static constexpr int kSmem = align16(kOffBars + kNBars * 8 + 16);
    __host__ __device__ static constexpr int box(int part, int stage) {
        return kOffRing + (part * kStages + stage) * kTcBox;
    }
};

// Byte offset of element (row, col) of a K-major operand with 64 columns
// (128-byte rows), 8-row swizzle atoms of 1024 bytes: atom row group | row |
// 16-byte chunk ^ (row % 8).  Operand tiles start on 1024-byte boundaries.
__device__ __forceinline__ int sw128_offset(int row, int col) {
    return (row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2;
}

// Query slot layout: `rows` rows x 128 columns as two 64-column halves.
__device__ __forceinline__ int qslot_offset(int row, int col, int rows) {
    return (col >> 6) * rows * 128 + sw128_offset(row, col & 63);
}

// Reduce v[0..15] over the warp's 32 lanes (max or sum), scattered: lane l
// ends with the result of row (l >> 1) & 15.  A butterfly that halves the
// vector at offsets 16, 8, 4, 2 (each lane keeps the half named by its offset
// bit) and a final exchange at offset 1: 16 shuffles for 16 rows.  v is
// consumed.
template <bool MAX>
__device__ __forceinline__ float warp_reduce_scatter16(float (&v)[16]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 4; ++step) {
        const int off = 16 >> step, half = 8 >> step;
        const bool up = lane & off;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    const float got = __shfl_xor_sync(0xffffffffu, v[0], 1);
    return MAX ? fmaxf(v[0], got) : v[0] + got;
}

// c ? x : y through an opaque select, so that a chain of them over an array
// indexed by constants is not folded into one dynamically indexed load
// (which would move the array to local memory).
__device__ __forceinline__ float select_f(bool c, float x, float y) {
    float r;
    asm("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %3, 0;\n\tselp.f32 %0, %1, %2, p;\n\t}"
        : "=f"(r)
        : "f"(x), "f"(y), "r"((unsigned)c));
    return r;
}

// RQ: query rows the softmax warps process (rows rounded up to 4, 8 or 16);
// P rows beyond RQ stay zero.
template <int RQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, AttnArgs a) {
    static_assert(RQ == 4 || RQ == 8 || RQ == 16, "row counts");
    constexpr int NQ = kTcNQ;
    using TL = TcLayout<RQ>;
    constexpr int kStages = TL::kStages;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *pbuf = smem + TL::kOffP;
    uint8_t *qslots = smem + TL::kOffQ;
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + TL::kOffMeta);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TL::kOffBars);
    uint64_t *full = bars;                       // [kStages] tile landed
    uint64_t *empty = full + kStages;            // [kStages] products done with the stage
    uint64_t *s_full = empty + kStages;          // [pair * 2 + buffer] S computed
    uint64_t *s_free = s_full + 4;               // [pair * 2 + buffer] S read
    uint64_t *p_full = s_free + 4;               // [2 pairs] P written (and V tail zeroed)
    uint64_t *pv_done = p_full + 2;              // [2] the pair's latest PV product completed
    uint64_t *fin = pv_done + 2;                 // MMA issuer: all products completed
    uint64_t *done = fin + 1;                    // softmax warps finished with TMEM
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    constexpr uint32_t kIdescQK = umma_idesc_bf16(128, NQ, false, false);
    constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 128, false, true);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int p = 0; p < 4; ++p) {
            mbar_init(&s_full[p], 1);
            mbar_init(&s_free[p], 2);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&p_full[p], 2);
            mbar_init(&pv_done[p], 1);
        }
        mbar_init(fin, 1);
        mbar_init(done, 4);
        fence_mbar_init();
    }
    // P starts zero: each warp only ever writes its own rows at its own tokens
    for (int i = threadIdx.x; i < 128 * 128 / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(pbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    // the lines (and translations) of the selection, the table and the
    // lengths; prefetches use no data, so they may precede the wait
    if (warp == 4) {
        const int64_t nsel = (int64_t)(a.units / a.ntiles) * a.max_sel;
        const int64_t nbt = (int64_t)(a.units / (a.ntiles * a.hkv)) * a.max_blocks;
        const void *p[6] = {a.sel_count, a.sel_idx, a.sel_idx + (nsel > 0 ? nsel - 1 : 0), a.block_table,
                            a.block_table + (nbt > 0 ? nbt - 1 : 0), a.seq_lens};
        if (lane < 6) prefetch_l2(p[lane]);
    }
    // Launched early (programmatic dependent launch): nothing above reads
    // global memory, as every input may come from the kernel before.  Once
    // the wait returns, that kernel's writes (the selection) are final, so
    // the merge behind this kernel may be scheduled: it reads only the
    // selection counts before its own wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 4) {
        // ============================================================ producer
        const uint64_t kv_policy = l2_evict_first();
        int64_t W = 0;
        for (int u0 = 0; u0 < a.units; u0 += 32) {
            const int u = u0 + lane;
            W += (u < a.units) ? unit_count(a, u) : 0;
        }
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        const int64_t lo = W * c / C, hi = W * (c + 1) / C;
        int i_push = 0, seg = -1, qs = 0;   // seg: current segment id, qs: its query slot
        int prev_seg = -1, prev_page = -1;  // the tile pushed last
        constexpr int kQTasks = TL::kQRows * 16 / 32;
        uint4 qreg[kQTasks];                // this lane's share of the next segment's query rows
        // Push one stage (whole warp, uniformly): wait for the stage, write the
        // query slot at a segment start, then lane 0 writes the stage's meta
        // and issues the TMA copies.  Block index and page come in resolved,
        // so no global load sits between the wait and the copy.
        auto push = [&](int unit, int j, int page, int flags) -> bool {
            const int s = i_push % kStages;
            int okw = 1;
            if (lane == 0 && i_push >= kStages)
                okw = mbar_wait(&empty[s], ((i_push / kStages) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
            if (flags & kFirst) {
                // the stage is free, so the segment that last used this slot is done
                ++seg;
                qs = seg % kStages;
                uint8_t *qd = qslots + qs * TL::kQSlot;
#pragma unroll
                for (int e = 0; e < kQTasks; ++e) {
                    const int task = lane + 32 * e, row = task >> 4, c8 = task & 15;
                    *reinterpret_cast<uint4 *>(qd + qslot_offset(row, c8 * 8, TL::kQRows)) = qreg[e];
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            // an odd tile of the same segment as the even one before it, both
            // loaded: one S product for the two
            const bool joint = (i_push & 1) && !(flags & kEnd) && page >= 0 && prev_page >= 0 && prev_seg == seg;
            if (lane == 0) {
                meta[s] = StageMeta{j, page, unit, flags | (joint ? kJoint : 0), seg, 0, qs, 0};
                if (page >= 0) {
                    const int y = (page * a.hkv + unit % a.hkv) * kBlock;
                    mbar_arrive_expect_tx(&full[s], kTcStageBytes);
                    tma_load_2d(smem + TL::box(0, s), &kmap, 0, y, &full[s], kv_policy);
                    tma_load_2d(smem + TL::box(1, s), &kmap, 64, y, &full[s], kv_policy);
                    tma_load_2d(smem + TL::box(2, s), &vmap, 0, y, &full[s], kv_policy);
                    tma_load_2d(smem + TL::box(3, s), &vmap, 64, y, &full[s], kv_policy);
                } else {
                    mbar_arrive(&full[s]);
                }
            }
            prev_page = (flags & kEnd) ? -1 : page;
            prev_seg = seg;
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
                const int b = unit / a.hkv, h = unit % a.hkv;
                const int ia = (int)(lo > us ? lo - us : 0);
                const int ib = (int)(hi - us < uc ? hi - us : uc);
                const int32_t *sel = a.sel_idx + (int64_t)unit * a.max_sel;
                // the segment's query rows (bf16 as stored, zero padded), into registers now
#pragma unroll
                for (int e = 0; e < kQTasks; ++e) {
                    const int task = lane + 32 * e, row = task >> 4, c8 = task & 15;
                    qreg[e] = make_uint4(0u, 0u, 0u, 0u);
                    if (row < a.rows) {
                        const int t = row / a.group, g = row % a.group;
                        qreg[e] = *reinterpret_cast<const uint4 *>(
                            a.q + (((int64_t)b * a.tq + t) * a.hq + h * a.group + g) * kHeadDim + c8 * 8);
                    }
                }
                int L = a.seq_lens[b];
                L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
                const int nb = (L + kBlock - 1) / kBlock;
                for (int i0 = ia; i0 < ib && ok; i0 += 32) {
                    // lane l resolves tile i0 + l: block index and page, checked
                    // (the table load does not wait for the length check)
                    int jl = 0, pl = -1;
                    if (i0 + lane < ib) {
                        jl = sel[i0 + lane];
                        const bool in_table = jl >= 0 && jl < a.max_blocks;
                        const int pg = in_table ? a.block_table[(int64_t)b * a.max_blocks + jl] : -1;
                        if (!in_table || jl >= nb)
                            flag(SPATTN_DEV_BAD_BLOCK);
                        else if (pg < 0 || pg >= a.num_pages)
                            flag(SPATTN_DEV_BAD_PAGE);
                        else
                            pl = pg;
                    }
                    const int n_here = ib - i0 < 32 ? ib - i0 : 32;
                    for (int e = 0; e < n_here && ok; ++e) {
                        const int i = i0 + e;
                        ok = push(unit, __shfl_sync(0xffffffffu, jl, e), __shfl_sync(0xffffffffu, pl, e),
                                  (i == ia ? kFirst : 0) | (i == ib - 1 ? kLast : 0));
                    }
                }
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        // one end marker for each pair
        if (ok) ok = push(0, 0, -1, kEnd);
        if (ok) push(0, 0, -1, kEnd);
        if (lane == 0) {
            for (int i = max(0, i_push - kStages); i < i_push; ++i)
                mbar_wait(&full[i % kStages], (i / kStages) & 1);
        }
        return;
    }

    if (warp == 5) {
        // ============================================================ MMA issue
        // PV products in tile order, each as soon as its P is written (it
        // releases a stage for the next copy); QK products run ahead as far
        // as stages and S buffers allow.  Non-blocking polls (test_wait,
        // which never suspends), so a tile still in flight never holds back
        // a product that is ready.
        if (lane == 0) {
            int qk = 0, pv = 0, n = 0x7fffffff;
            int last_seg0 = -1, last_seg1 = -1;   // segment of each pair's latest PV product
            bool idle = false;
            uint64_t t_idle = 0;
            // S^T = K . Q^T over d in 8 steps of 16; K rows from the K boxes at
            // k0 / k1 (d 0-63 / 64-127, 128 rows each), Q from query slot qslot
            auto issue_qk = [&](uint32_t k0, uint32_t k1, int qslot, uint32_t d) {
                const uint32_t qb = smem_u32(qslots + qslot * TL::kQSlot);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = sw128_desc((ks < 4 ? k0 : k1) + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(qb + (ks >> 2) * TL::kQRows * 128 + (ks & 3) * 32, 16, 1024);
                    umma_bf16(d, ad, bd, kIdescQK, ks > 0);
                }
            };
            while (pv < n) {
                bool progressed = false;
                if (pv < (2 * qk < n ? 2 * qk : n)) {   // first: a PV product frees a stage
                    const int s = pv % kStages, p = pv & 1;
                    if (mbar_test_wait(&p_full[p], (pv >> 1) & 1)) {
                        tc_fence_after();
                        const StageMeta m = meta[s];
                        if (m.page >= 0) {
                            const uint32_t acc0 = (p ? last_seg1 : last_seg0) == m.seg ? 1u : 0u;
                            if (p)
                                last_seg1 = m.seg;
                            else
                                last_seg0 = m.seg;
                            const uint32_t vb = smem_u32(smem + TL::box(2, s));
                            const uint32_t pb = smem_u32(pbuf);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                const uint64_t ad = sw128_desc(pb + ks * 32, 16, 1024);
                                const uint64_t bd = sw128_desc(vb + ks * 2048, TL::box(3, 0) - TL::box(2, 0), 1024);
                                umma_bf16(tbase + 4 * NQ + p * 128, ad, bd, kIdescPV, ks > 0 ? 1u : acc0);
                            }
                            umma_commit(&pv_done[p]);
                            umma_commit(&empty[s]);
                        } else {
                            mbar_arrive(&pv_done[p]);
                            mbar_arrive(&empty[s]);
                        }
                        ++pv;
                        progressed = true;
                    }
                }
                if (2 * qk < n) {
                    // S of tiles t0 = 2 qk (pair 0) and t1 = t0 + 1 (pair 1), into S
                    // buffer j of each pair; that buffer's previous use (the
                    // pairs' tiles of qk - 2) must have been read by both pairs
                    const int t0 = 2 * qk, t1 = t0 + 1, s0 = t0 % kStages, s1 = t1 % kStages, j = qk & 1;
                    if (mbar_test_wait(&full[s0], (t0 / kStages) & 1) &&
                        mbar_test_wait(&full[s1], (t1 / kStages) & 1) &&
                        (qk < 2 || (mbar_test_wait(&s_free[j], ((qk >> 1) - 1) & 1) &&
                                    mbar_test_wait(&s_free[2 + j], ((qk >> 1) - 1) & 1)))) {
                        const StageMeta m0 = meta[s0], m1 = meta[s1];
                        if (m0.flags & kEnd) {
                            n = t0;
                        } else {
                            tc_fence_after();
                            // rows 0-63 from stage s0's K boxes, 64-127 from the next stage's
                            const uint32_t k0 = smem_u32(smem + TL::box(0, s0)), k1 = smem_u32(smem + TL::box(1, s0));
                            if (m1.flags & kJoint) {
                                issue_qk(k0, k1, m0.qslot, tbase + j * NQ);
                                umma_commit(&s_full[j]);
                                umma_commit(&s_full[2 + j]);
                            } else {
                                if (m0.page >= 0) {
                                    issue_qk(k0, k1, m0.qslot, tbase + j * NQ);
                                    umma_commit(&s_full[j]);
                                } else {
                                    mbar_arrive(&s_full[j]);
                                }
                                if (m1.flags & kEnd) {
                                    n = t1;
                                } else if (m1.page >= 0) {
                                    // the odd tile alone: start 64 rows early so its rows are 64-127
                                    issue_qk(k0, k1, m1.qslot, tbase + (2 + j) * NQ);
                                    umma_commit(&s_full[2 + j]);
                                } else {
                                    mbar_arrive(&s_full[2 + j]);
                                }
                            }
                            ++qk;
                        }
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = false;
                } else if (!idle) {
                    idle = true;
                    t_idle = global_ns();
                } else if (global_ns() - t_idle > kWaitLimitNs) {
                    flag(SPATTN_DEV_WAIT_TIMEOUT);
                    break;
                }
            }
            // every product issued has completed before TMEM can go
            umma_commit(fin);
            mbar_wait(fin, 0);
        }
        __syncwarp();
        mbar_wait(done, 0);
        tc_fence_after();
        tmem_dealloc(tbase, kTcTmemCols);
        return;
    }

    // ==================================================== softmax (warps 0-3)
    const int pr = warp >> 1;                    // pair: even or odd tiles
    const int tok = (warp & 1) * 32 + lane;      // this lane's token of the block
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    const uint32_t s_tm = tbase + lanes;                    // + S buffer column
    const uint32_t o_tm = tbase + lanes + 4 * NQ + pr * 128;

    float m_ref[RQ], l_run[RQ];
    int cur_seg = -1, unit = 0, L = 0, k_last = -1;
    bool had_pv = false;   // a PV product of this segment has written this warp's lanes

    for (int k = 0;; ++k) {
        const int i = 2 * k + pr, s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1)) break;
        const StageMeta md = meta[s];
        const bool end = md.flags & kEnd;
        if (cur_seg >= 0 && (end || md.seg != cur_seg)) {
            // ---- end of this warp's share of a segment: its partial record (m, l, O)
            if (k_last >= 0 && !mbar_wait(&pv_done[pr], k_last & 1)) break;
            tc_fence_after();
            float v16[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) v16[r] = r < RQ ? l_run[r] : 0.f;
            const float ls = warp_reduce_scatter16<false>(v16);
            const float l_row = __shfl_sync(0xffffffffu, ls, 2 * (lane & 15));
            float m_row = -INFINITY;
#pragma unroll
            for (int r = 0; r < RQ; ++r) m_row = select_f((lane & 15) == r, m_ref[r], m_row);
            const int64_t rec = (((int64_t)c + unit) * kTcWarpSlots + warp) * a.rows;
            const uint64_t keep = l2_evict_last();   // the merge reads the record next
            if (lane < a.rows) st_global_f2(a.part_ml + (rec + lane) * 2, m_row, l_row, keep);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float v[16];
                if (had_pv) {
                    tmem_ld16(o_tm + cc * 16, v);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] += __shfl_xor_sync(0xffffffffu, v[e], 16);   // hi + lo
                if (lane < a.rows) {
                    float *dst = a.part_o + (rec + lane) * kHeadDim + cc * 16;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        st_global_f4(dst + 4 * e, v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3], keep);
                }
            }
            tc_fence_before();
            cur_seg = -1;
        }
        if (end) break;
        if (cur_seg < 0) {
            cur_seg = md.seg;
            unit = md.unit;
            L = a.seq_lens[unit / a.hkv];
            L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
            had_pv = false;
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                m_ref[r] = -INFINITY;
                l_run[r] = 0.f;
            }
        }
        const bool valid = md.page >= 0;
        const int pos = md.j * kBlock + tok;
        // ---- scores of this lane's token, in log2 units, masked
        const int sb = 2 * pr + (k & 1);
        if (!mbar_wait(&s_full[sb], (k >> 1) & 1)) break;
        tc_fence_after();
        float x[RQ];
        if (valid) {
            float sv[16];
            // pair 0's S in buffer k & 1; pair 1's beside it, or in pair 0's
            // columns (its lanes 64-127) when the two tiles shared a product
            tmem_ld16(s_tm + ((pr && !(md.flags & kJoint)) ? 2 + (k & 1) : (k & 1)) * NQ, sv);
            // row r (chunk token r / group at position L - tq + r / group)
            // sees pos when pos < L and r >= rmin
            const int ahead = pos - (L - a.tq);
            const int rmin = pos >= L ? NQ : (ahead <= 0 ? 0 : ahead * a.group);
#pragma unroll
            for (int r = 0; r < RQ; ++r) x[r] = (r >= rmin && r < a.rows) ? sv[r] * a.qscale : -INFINITY;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        // ---- the pair's previous product is done: P rows free, O settled
        if (k > 0 && !mbar_wait(&pv_done[pr], (k - 1) & 1)) break;
        tc_fence_after();
        if (valid) {
            float over = -INFINITY;
#pragma unroll
            for (int r = 0; r < RQ; ++r) over = fmaxf(over, x[r] - m_ref[r]);   // NaN (both -inf) is ignored
            if (__any_sync(0xffffffffu, over > kTcSlack)) {
                // rebase: reference = max(reference, block maximum) per row
                float v16[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) v16[r] = r < RQ ? x[r] : -INFINITY;
                const float mx = warp_reduce_scatter16<true>(v16);
                float al = 1.f;   // the factor of this lane's accumulator row
#pragma unroll
                for (int r = 0; r < RQ; ++r) {
                    const float m_new = fmaxf(m_ref[r], __shfl_sync(0xffffffffu, mx, 2 * r));
                    const float alpha = m_new == m_ref[r] ? 1.f : exp2f(m_ref[r] - m_new);
                    m_ref[r] = m_new;
                    l_run[r] *= alpha;
                    al = select_f((lane & 15) == r, alpha, al);
                }
                if (had_pv) {
#pragma unroll 1
                    for (int cc = 0; cc < 8; ++cc) {
                        float v[16];
                        tmem_ld16(o_tm + cc * 16, v);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= al;
                        tmem_st16(o_tm + cc * 16, v);
                    }
                    tmem_wait_st();
                }
            }
            // ---- weights into P (hi and lo rows), running sums per lane
#pragma unroll
            for (int r = 0; r < RQ; ++r) {
                const float mu = m_ref[r] == -INFINITY ? 0.f : m_ref[r];
                const float p = exp2f(x[r] - mu);
                l_run[r] += p;
                const __nv_bfloat16 h = __float2bfloat16_rn(p);
                const __nv_bfloat16 l = __float2bfloat16_rn(p - __bfloat162float(h));
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + sw128_offset(warp * 32 + r, tok)) = h;
                *reinterpret_cast<__nv_bfloat16 *>(pbuf + sw128_offset(warp * 32 + 16 + r, tok)) = l;
            }
            if (pos >= L) {
                // unfilled slot: its V row must be finite under the zero weights
                uint4 *v0 = reinterpret_cast<uint4 *>(smem + TL::box(2, s) + tok * 128);
                uint4 *v1 = reinterpret_cast<uint4 *>(smem + TL::box(3, s) + tok * 128);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v0[e] = make_uint4(0u, 0u, 0u, 0u);
                    v1[e] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            had_pv = true;
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pr]);
        k_last = k;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(done);
}

}  // namespace spattn
