// attention_tcw.cuh -- exact softmax attention over the kept blocks on the
// sm_100a tensor cores for many query rows per KV head (a chunk of tokens
// times the group's heads, up to 64) and for fp8 caches.
//
// "CSA + HCA 混合注意力机制" §2.1 / §4.4 step 4: softmax(q K_sel^T / sqrt(d)) V_sel
// over the selected entries only; §4.3: the window and the partly filled
// tail join the same softmax.  "Claude Code 1M 上下文" §2(3): K and V may be
// stored as fp8 with a scale per (page, KV head).
//
// Work split, segments and records follow attention.cuh: the kept lists of
// all (request, KV head) units are concatenated and cut into equal ranges,
// one per CTA of a persistent grid.
//
// Products per kept block (64 tokens), query rows on M:
//   S [128 x 64]   = Q [128 x d] . K^T      K-major A (query slot) and B (the
//                    block's keys).  Rows 0-63 are the unit's query rows
//                    (zero padded); rows 64-127 read whatever follows the
//                    slot and are never used.
//   O_hi [128 x d] += P [128 x 64] . V      K-major A, MN-major B.  Row r of
//   O_lo [128 x d] += P' [128 x 64] . V     P holds hi(p_r) (p truncated to
//                    bf16) for query row r, row 64 + r the remainder lo(p_r) =
//                    p - hi, truncated to bf16 (~15 significant bits
//                    together); P' is P from row 64 on.  Lanes 0-63 of the
//                    two accumulators (separate TMEM columns) are the two
//                    parts of each row's output; the other lanes are never
//                    read.  P is double buffered, so the weights of a block
//                    are written while the previous block's products run.
// Each softmax thread owns one query row: its scores come from its own TMEM
// lane, the row maximum is thread-local, and it keeps a reference maximum
// raised only when a score exceeds it by kTcSlack (then both parts of its O
// row are rescaled).  One partial record (m, l, O = hi + lo) per row and
// segment.
//
// fp8 caches: the bulk copies land in a staging buffer and converter warps
// widen the codes to bf16 (exact: every e4m3 value is a bf16 value) into the
// operand layout; the per-(page, KV head) scales multiply the scores (K) and
// the weights (V).  bf16 caches are copied straight into the operand layout
// by TMA.  Either way the converter warps zero the V rows of unfilled token
// slots, so that zero weights never meet non-finite values.
//
// Warps: 0-1 softmax (query rows 0-63; TMEM lanes 0-63), 4 producer, 5 MMA
// issue (one lane) and TMEM owner, 2, 3, 6, 7 converters.  Every wait is
// bounded (SPATTN_DEV_WAIT_TIMEOUT).
#pragma once

#include "attention.cuh"
#include "attention_tc.cuh"
#include "tcgen05.cuh"

namespace spattn {

// 8 warps; warp w runs on SM sub-partition w % 4.  The softmax warps (0, 1)
// share sub-partitions 0 and 1 only with the producer and the MMA issuer;
// the converters (warps 2, 3, 6, 7) have sub-partitions 2 and 3 to
// themselves.  Two warps per sub-partition leave room for 255 registers.
constexpr int kTcwThreads = 8 * 32;
constexpr int kTcwRows = 64;                  // query rows per unit, at most
constexpr int kTcwConvWarps = 4;
__device__ __forceinline__ int tcw_conv_index(int warp) {   // 0..3 for a converter warp, else -1
    return warp == 2 ? 0 : warp == 3 ? 1 : warp == 6 ? 2 : warp == 7 ? 3 : -1;
}
constexpr int kTcwTmemCols = 512;             // S: 2 x 64 | O hi: 128 | O lo: 128
constexpr int kTcwOHi = 128, kTcwOLo = 256;   // TMEM columns of the two output parts

struct TcwMeta {
    int j;         // logical block id
    int page;      // -1 when the block or its page is invalid
    int unit;
    int flags;     // kFirst | kLast | kEnd
    int seg;
    int nvalid;    // filled token slots of the block
    int qslot;
    float ks, vs;  // the block's K and V scales (1 for bf16 caches)
    int pad[3];
};

// Shared memory: two query slots (64 rows x 128 bf16 as two 64-column halves),
// two P buffers (128 rows x 64 bf16), per stage the K and V operands (two
// 64 x 64 bf16 boxes each) and, for fp8, the staging of the copied codes;
// then meta and barriers.  Operand tiles on 1024-byte boundaries.  (A
// separate, deeper staging ring released at conversion measured slower: the
// converters then wait on the products instead of on the copies.)
template <bool FP8>
struct TcwLayout {
    static constexpr int kOp = FP8 ? 3 : 4;          // stages (bf16 K and V operands of a block)
    static constexpr int kStg = FP8 ? kOp : 0;       // fp8: the staging buffer of each stage
    static constexpr int kSrc = kOp;                 // the ring the copies land in
    static constexpr int kMeta = kOp;                // tiles in flight at most
    static constexpr int kQSlot = kTcwRows * 256;
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + 2 * kQSlot;                   // [2] P buffers
    static constexpr int kOffK = kOffP + 2 * 128 * 128;
    static constexpr int kOffV = kOffK + kOp * 16384;
    static constexpr int kOffStg = kOffV + kOp * 16384;                // fp8: [stage][K | V] codes
    static constexpr int kOffMeta = kOffStg + kStg * 16384;
    static constexpr int kNBars = 3 * kOp + 5 * 2 + 2;
    static constexpr int kOffBars = align16(kOffMeta + kMeta * (int)sizeof(TcwMeta));
    static constexpr int kSmem = align16(kOffBars + kNBars * 8 + 16);
};

// Two e4m3 codes (low byte first) -> two bf16 (low half first), exactly:
// the hardware e4m3x2 -> f16x2 conversion, then f16 -> bf16 by moving the
// fields (every e4m3 value is a normal f16 or zero, with at most 3 mantissa
// bits): magnitude >> 3 puts exponent and mantissa in place, + 112 << 7
// rebiases the exponent for the nonzero halves, and the sign stays.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t codes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(codes & 0xffffu)));
    const uint32_t mag = (h2 >> 3) & 0x0fff0fffu;               // 0, or >= 0x300 (2^-9) per half
    const uint32_t nz = ((mag + 0x0d000d00u) & 0x10001000u) >> 12;   // 1 per nonzero half
    return (nz * 0x3800u + mag) | (h2 & 0x80008000u);
}

// 2^x by the hardware approximation (relative error ~2^-22), results below
// the normal range flushed to zero: a weight that small is below the fp32
// resolution of the row sum, which is at least 1 (the maximum's own weight)
// or, before the row's first visible score, exactly 0.
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 64 consecutive 32-bit TMEM columns of this thread's lane, one load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

template <bool FP8>
__global__ void __launch_bounds__(kTcwThreads, 1)
    attn_tcw_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, AttnArgs a) {
    using TL = TcwLayout<FP8>;
    constexpr int kOp = TL::kOp, kSrc = TL::kSrc, kMeta = TL::kMeta;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *pbuf = smem + TL::kOffP;
    TcwMeta *meta = reinterpret_cast<TcwMeta *>(smem + TL::kOffMeta);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TL::kOffBars);
    uint64_t *full = bars;                      // [kOp] copies landed
    uint64_t *conv = full + kSrc;               // [kOp] operands ready (converters)
    uint64_t *empty = conv + kOp;               // [kOp] products done with the operand stage
    // per-buffer barriers ([k & 1] for tile k), so that no parity wait can
    // be lapped by a phase two tiles ahead
    uint64_t *s_full = empty + kOp;             // [2] S buffer computed
    uint64_t *s_free = s_full + 2;              // [2] S buffer read (warps 0, 1)
    uint64_t *p_full = s_free + 2;              // [2] P buffer written, rescales done (warps 0-3)
    uint64_t *pv_done = p_full + 2;             // [2] the PV product of that buffer completed
    uint64_t *q_free = pv_done + 2;             // [2] query slot's last product completed
    uint64_t *fin = q_free + 2;                 // MMA issuer: all products completed
    uint64_t *done = fin + 1;                   // warps 0-3 finished with TMEM
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 64, false, false);
    constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 128, false, true);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kOp; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], kTcwConvWarps);
            mbar_init(&empty[s], 1);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&s_full[p], 1);
            mbar_init(&s_free[p], 2);
            mbar_init(&q_free[p], 1);
            mbar_init(&p_full[p], 2);
            mbar_init(&pv_done[p], 1);
        }
        mbar_init(fin, 1);
        mbar_init(done, 2);
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTcwTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 4) {
        // ============================================================ producer
        int64_t W = 0;
        for (int u0 = 0; u0 < a.units; u0 += 32) {
            const int u = u0 + lane;
            W += (u < a.units) ? unit_count(a, u) : 0;
        }
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        const int64_t lo = W * c / C, hi = W * (c + 1) / C;
        int i_push = 0, seg = -1;
        // Push one stage (whole warp, uniformly): wait for the stage, at a
        // segment start wait for the query slot and fill it, then lane 0
        // writes the stage's meta and issues the copies.
        auto push = [&](int unit, int j, int page, int flags, int nvalid) -> bool {
            // the stage is free once its products are done
            const int s = i_push % kOp;
            int okw = 1;
            if (lane == 0 && i_push >= kOp) okw = mbar_wait(&empty[s], ((i_push / kOp) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
            int qs = seg & 1;
            if (flags & kFirst) {
                ++seg;
                qs = seg & 1;
                if (lane == 0 && seg >= 2) okw = mbar_wait(&q_free[qs], ((seg >> 1) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
                // the segment's query rows (bf16 as stored, zero padded)
                const int b = unit / a.hkv, h = unit % a.hkv;
                uint8_t *qd = smem + TL::kOffQ + qs * TL::kQSlot;
                for (int task = lane; task < kTcwRows * 16; task += 32) {
                    const int row = task >> 4, c8 = task & 15;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (row < a.rows) {
                        const int t = row / a.group, g = row % a.group;
                        v = *reinterpret_cast<const uint4 *>(
                            a.q + (((int64_t)b * a.tq + t) * a.hq + h * a.group + g) * kHeadDim + c8 * 8);
                    }
                    *reinterpret_cast<uint4 *>(qd + qslot_offset(row, c8 * 8, kTcwRows)) = v;
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                float ks = 1.f, vs = 1.f;
                if (FP8 && page >= 0) {
                    ks = a.k_scale[(int64_t)page * a.hkv + unit % a.hkv];
                    vs = a.v_scale[(int64_t)page * a.hkv + unit % a.hkv];
                }
                meta[i_push % kMeta] = TcwMeta{j, page, unit, flags, seg, nvalid, qs, ks, vs, {0, 0, 0}};
                if (page >= 0) {
                    const int y = (page * a.hkv + unit % a.hkv) * kBlock;
                    if (FP8) {
                        mbar_arrive_expect_tx(&full[s], 2 * 8192);
                        tma_load_2d(smem + TL::kOffStg + s * 16384, &kmap, 0, y, &full[s]);
                        tma_load_2d(smem + TL::kOffStg + s * 16384 + 8192, &vmap, 0, y, &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], 4 * 8192);
                        tma_load_2d(smem + TL::kOffK + s * 16384, &kmap, 0, y, &full[s]);
                        tma_load_2d(smem + TL::kOffK + s * 16384 + 8192, &kmap, 64, y, &full[s]);
                        tma_load_2d(smem + TL::kOffV + s * 16384, &vmap, 0, y, &full[s]);
                        tma_load_2d(smem + TL::kOffV + s * 16384 + 8192, &vmap, 64, y, &full[s]);
                    }
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
                const int b = unit / a.hkv;
                const int ia = (int)(lo > us ? lo - us : 0);
                const int ib = (int)(hi - us < uc ? hi - us : uc);
                const int32_t *sel = a.sel_idx + (int64_t)unit * a.max_sel;
                int L = a.seq_lens[b];
                L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
                const int nb = (L + kBlock - 1) / kBlock;
                for (int i0 = ia; i0 < ib && ok; i0 += 32) {
                    // lane l resolves tile i0 + l: block index and page, checked
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
                        const int j = __shfl_sync(0xffffffffu, jl, e);
                        const int nv = min(kBlock, max(0, L - j * kBlock));
                        ok = push(unit, j, __shfl_sync(0xffffffffu, pl, e),
                                  (i == ia ? kFirst : 0) | (i == ib - 1 ? kLast : 0), nv);
                    }
                }
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (ok) push(0, 0, -1, kEnd, 0);
        if (lane == 0) {
            for (int i = max(0, i_push - kSrc); i < i_push; ++i) mbar_wait(&full[i % kSrc], (i / kSrc) & 1);
        }
        return;
    }

    if (tcw_conv_index(warp) >= 0) {
        // ========================================================== converters
        // Stage by stage: fp8 codes -> bf16 operand boxes, V rows of unfilled
        // slots zeroed; then the operands are released to the MMA issuer.
        // Lanes take consecutive tokens of one 16-column chunk: both the
        // 128-byte-swizzled staging rows and the operand rows are then read
        // and written without bank conflicts.
        const int ct = tcw_conv_index(warp) * 32 + lane;   // 0 .. 32 * kTcwConvWarps - 1
        for (int i = 0;; ++i) {
            const int rs = i % kSrc, os = i % kOp;
            if (!mbar_wait(&full[rs], (i / kSrc) & 1)) break;
            const TcwMeta m = meta[i % kMeta];
            if (m.page >= 0) {
                uint8_t *kop = smem + TL::kOffK + os * 16384, *vop = smem + TL::kOffV + os * 16384;
                if (FP8) {
                    const uint8_t *stg = smem + TL::kOffStg + rs * 16384;
#pragma unroll
                    for (int e = 0; e < 1024 / (kTcwConvWarps * 32); ++e) {
                        const int task = ct + e * kTcwConvWarps * 32;
                        const bool isv = task >= 512;
                        const int tt = task & 63, c16 = (task >> 6) & 7;   // token, 16-column chunk
                        const uint4 u = *reinterpret_cast<const uint4 *>(stg + (isv ? 8192 : 0) + tt * 128 +
                                                                         ((c16 ^ (tt & 7)) << 4));
                        uint4 w0 = make_uint4(e4m3x2_to_bf16x2(u.x), e4m3x2_to_bf16x2(u.x >> 16),
                                              e4m3x2_to_bf16x2(u.y), e4m3x2_to_bf16x2(u.y >> 16));
                        uint4 w1 = make_uint4(e4m3x2_to_bf16x2(u.z), e4m3x2_to_bf16x2(u.z >> 16),
                                              e4m3x2_to_bf16x2(u.w), e4m3x2_to_bf16x2(u.w >> 16));
                        if (isv && tt >= m.nvalid) w0 = w1 = make_uint4(0u, 0u, 0u, 0u);
                        uint8_t *box = (isv ? vop : kop) + (c16 >> 2) * 8192;
                        const int col = (c16 & 3) * 16;
                        *reinterpret_cast<uint4 *>(box + sw128_offset(tt, col)) = w0;
                        *reinterpret_cast<uint4 *>(box + sw128_offset(tt, col + 8)) = w1;
                    }
                } else if (m.nvalid < kBlock) {
                    for (int task = ct; task < (kBlock - m.nvalid) * 16; task += kTcwConvWarps * 32) {
                        const int tt = m.nvalid + (task >> 4), c8 = task & 15;
                        *reinterpret_cast<uint4 *>(vop + (c8 >> 3) * 8192 + sw128_offset(tt, (c8 & 7) * 8)) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[os]);
            if (m.flags & kEnd) break;
        }
        return;
    }

    if (warp == 5) {
        // ============================================================ MMA issue
        if (lane == 0) {
            int qk = 0, pv = 0, n = 0x7fffffff, last_seg = -1;
            bool idle = false;
            uint64_t t_idle = 0;
            while (pv < n) {
                bool progressed = false;
                if (pv < qk && mbar_test_wait(&p_full[pv & 1], (pv >> 1) & 1)) {   // first: a PV product frees a stage
                    tc_fence_after();
                    const int s = pv % kOp;
                    const TcwMeta m = meta[pv % kMeta];
                    if (m.page >= 0) {
                        const uint32_t acc0 = last_seg == m.seg ? 1u : 0u;
                        last_seg = m.seg;
                        const uint32_t vb = smem_u32(smem + TL::kOffV + s * 16384);
                        const uint32_t pb = smem_u32(pbuf + (pv & 1) * 16384);
                        // O hi += P rows 0-63 . V ; O lo += P rows 64-127 . V (the
                        // other 64 lanes of each product are never read)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t bd = sw128_desc(vb + ks * 2048, 8192, 1024);
                            umma_bf16(tbase + kTcwOHi, sw128_desc(pb + ks * 32, 16, 1024), bd, kIdescPV,
                                      ks > 0 ? 1u : acc0);
                            umma_bf16(tbase + kTcwOLo, sw128_desc(pb + 8192 + ks * 32, 16, 1024), bd, kIdescPV,
                                      ks > 0 ? 1u : acc0);
                        }
                        umma_commit(&pv_done[pv & 1]);
                        umma_commit(&empty[s]);
                    } else {
                        mbar_arrive(&pv_done[pv & 1]);
                        mbar_arrive(&empty[s]);
                    }
                    ++pv;
                    progressed = true;
                }
                if (qk < n) {
                    const int s = qk % kOp, j = qk & 1;
                    if (mbar_test_wait(&conv[s], (qk / kOp) & 1) &&
                        (qk < 2 || mbar_test_wait(&s_free[j], ((qk >> 1) - 1) & 1))) {
                        const TcwMeta m = meta[qk % kMeta];
                        if (m.flags & kEnd) {
                            n = qk;
                        } else {
                            tc_fence_after();
                            if (m.page >= 0) {
                                const uint32_t qb = smem_u32(smem + TL::kOffQ + m.qslot * TL::kQSlot);
                                const uint32_t kb = smem_u32(smem + TL::kOffK + s * 16384);
#pragma unroll
                                for (int ks = 0; ks < 8; ++ks) {
                                    const uint64_t ad = sw128_desc(qb + (ks >> 2) * (kTcwRows * 128) + (ks & 3) * 32, 16, 1024);
                                    const uint64_t bd = sw128_desc(kb + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                                    umma_bf16(tbase + j * 64, ad, bd, kIdescQK, ks > 0);
                                }
                                umma_commit(&s_full[j]);
                            } else {
                                mbar_arrive(&s_full[j]);
                            }
                            // the slot is free once the segment's last product is done
                            if (m.flags & kLast) umma_commit(&q_free[m.qslot]);
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
                } else {
                    __nanosleep(32);   // leave the issue slots to the softmax warp sharing this SM sub-partition
                }
            }
            umma_commit(fin);
            mbar_wait(fin, 0);
        }
        __syncwarp();
        mbar_wait(done, 0);
        tc_fence_after();
        tmem_dealloc(tbase, kTcwTmemCols);
        return;
    }

    // ============================================== softmax (warps 0, 1)
    const int r = warp * 32 + lane;                       // query row (TMEM lane)
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    const int t_r = r / a.group;                          // the row's chunk token
    const bool row_ok = r < a.rows;

    float m_ref = -INFINITY, l_run = 0.f;
    int cur_seg = -1, unit = 0, L = 0, k_last = -1;
    bool had_pv = false;
    // wait for tile kk's PV products (its buffer's barrier)
    auto wait_pv = [&](int kk) -> bool { return mbar_wait(&pv_done[kk & 1], (kk >> 1) & 1); };
    auto rescale_o = [&](float f) {   // both parts of this row's accumulator
#pragma unroll 1
        for (int cc = 0; cc < 16; ++cc) {
            const uint32_t col = (cc < 8 ? kTcwOHi : kTcwOLo) + (cc & 7) * 16;
            float v[16];
            tmem_ld16(tbase + lanes + col, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= f;
            tmem_st16(tbase + lanes + col, v);
        }
        tmem_wait_st();
    };

    for (int k = 0;; ++k) {
        // operands of tile k ready (also publishes its meta)
        if (!mbar_wait(&conv[k % kOp], (k / kOp) & 1)) break;
        const TcwMeta md = meta[k % kMeta];
        const bool end = md.flags & kEnd;
        if (cur_seg >= 0 && (end || md.seg != cur_seg)) {
            // ---- end of a segment: this row's partial record (m, l, O = hi + lo)
            if (k_last >= 0 && !wait_pv(k_last)) break;
            tc_fence_after();
            const int64_t rec = ((int64_t)c + unit) * a.rows + r;
            if (row_ok) *reinterpret_cast<float2 *>(a.part_ml + rec * 2) = make_float2(m_ref, l_run);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float v[16], w[16];
                if (had_pv) {
                    tmem_ld16(tbase + lanes + kTcwOHi + cc * 16, v);
                    tmem_ld16(tbase + lanes + kTcwOLo + cc * 16, w);
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] += w[e];
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0.f;
                }
                if (row_ok) {
                    float4 *dst = reinterpret_cast<float4 *>(a.part_o + rec * kHeadDim + cc * 16);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
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
            m_ref = -INFINITY;
            l_run = 0.f;
        }
        const bool valid = md.page >= 0;
        const int j = k & 1;
        // ---- this row's 64 scores (one TMEM load), log2 units, masked
        if (!mbar_wait(&s_full[j], (k >> 1) & 1)) break;
        tc_fence_after();
        float x[64];
        if (valid) tmem_ld64(tbase + lanes + j * 64, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[j]);
        float alpha = 1.f;
        uint32_t hw[32], lw[32];
        if (valid) {
            const int lim = min(L - 1, L - a.tq + t_r);   // last position the row sees
            const float sc = a.qscale * md.ks;
            const int pos0 = md.j * kBlock;
            float mx = -INFINITY;
            if (row_ok && pos0 + 63 <= lim) {   // the whole block is visible to the row
#pragma unroll
                for (int t = 0; t < 64; ++t) {
                    x[t] *= sc;
                    mx = fmaxf(mx, x[t]);
                }
            } else {
#pragma unroll
                for (int t = 0; t < 64; ++t) {
                    x[t] = (row_ok && pos0 + t <= lim) ? x[t] * sc : -INFINITY;
                    mx = fmaxf(mx, x[t]);
                }
            }
            if (mx > m_ref + kTcSlack || (m_ref == -INFINITY && mx != -INFINITY)) {
                alpha = m_ref == -INFINITY ? 0.f : exp2f(m_ref - mx);
                m_ref = mx;
                l_run *= alpha;
            }
            // weights times the V scale, exp2(x - m + log2 vs), as bf16 hi / lo
            // pairs, ready before the buffer is waited for; the row sum is
            // taken over the scaled weights and divided by the scale once
            const float mu = (m_ref == -INFINITY ? 0.f : m_ref) - (md.vs == 1.f ? 0.f : __log2f(md.vs));
            float ps = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = ex2_ftz(x[2 * e] - mu), p1 = ex2_ftz(x[2 * e + 1] - mu);
                ps += p0 + p1;
                // hi = p with its low 16 bits cleared (a bf16 value), lo = the
                // exact fp32 remainder, truncated the same way: the pair keeps
                // ~15 significant bits, with integer ops only (the exp2 pipe
                // stays free for the exponentials)
                const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                const float r0 = p0 - __uint_as_float(b0 & 0xffff0000u);
                const float r1 = p1 - __uint_as_float(b1 & 0xffff0000u);
                hw[e] = __byte_perm(b0, b1, 0x7632);
                lw[e] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
            }
            l_run += md.vs == 1.f ? ps : ps / md.vs;
        }
        const float a_o = (valid && had_pv) ? alpha : 1.f;
        // ---- P buffer j is free once tile k - 2's products are done
        if (k >= 2 && !wait_pv(k - 2)) break;
        if (valid) {
            if (a_o != 1.f) {
                // rescale this row's accumulator: after tile k - 1's products
                if (k >= 1 && !wait_pv(k - 1)) break;
                tc_fence_after();
                rescale_o(a_o);
            }
            uint8_t *pb = pbuf + j * 16384;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                *reinterpret_cast<uint4 *>(pb + sw128_offset(r, c8 * 8)) =
                    make_uint4(hw[4 * c8], hw[4 * c8 + 1], hw[4 * c8 + 2], hw[4 * c8 + 3]);
                *reinterpret_cast<uint4 *>(pb + sw128_offset(64 + r, c8 * 8)) =
                    make_uint4(lw[4 * c8], lw[4 * c8 + 1], lw[4 * c8 + 2], lw[4 * c8 + 3]);
            }
            fence_proxy_async_smem();
            had_pv = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[j]);
        k_last = k;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(done);
}

}  // namespace spattn
