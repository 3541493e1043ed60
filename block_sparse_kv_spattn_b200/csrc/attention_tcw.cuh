// attention_tcw.cuh -- exact softmax attention over the kept blocks on the
// sm_100a tensor cores for many query rows per KV head (a chunk of tokens
// times the group's heads, in tiles of 64 rows) and for fp8 caches.
//
// "CSA + HCA 混合注意力机制" §2.1 / §4.4 step 4: softmax(q K_sel^T / sqrt(d)) V_sel
// over the selected entries only; §4.3: the window and the partly filled
// tail join the same softmax.  "Claude Code 1M 上下文" §2(3): K and V may be
// stored as fp8 with a scale per (page, KV head).
//
// Work split, segments and records follow attention.cuh: the kept lists of
// all units are concatenated and cut into equal ranges, one per CTA of a
// persistent grid; a unit is one 64-row tile of a (request, KV head), so a
// longer chunk runs as several units over the same kept blocks, each masked
// by its own rows' tokens.
//
// Products per kept block (64 tokens), query rows on M, bf16 caches:
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
// fp8 caches: the copies land in a ring of [K codes | V codes] stages.  The
// QK product runs in kind::f8f6f4 on the key codes as copied: each query row
// is scaled by a power of two (its largest element in [2^7, 2^8)) and split
// into two e4m3 terms q1 + q2, exact for every element within 2^9 of the
// row's largest, so S = q1 . K + q2 . K (the slot holds each term's 64 rows
// twice, rows r and 64 + r, so lanes 64-127 carry the same scores).
// Converter warps widen the V codes to f16 (exact) into their own buffers,
// and PV runs in f16 with one f16 weight per element (the reference maximum
// follows x + log2 s_v, so every weight stays below 2^15).  The softmax runs
// in two halves (tokens 0-31 and 32-63 of a block), each with its own
// reference maximum, sums, output rows and partial record.  The per-(page,
// KV head) scales multiply the scores (K) and the weights (V).  bf16 caches
// are copied straight into the operand layout by TMA.  Either way the
// converter warps zero the V rows of unfilled token slots, so that zero
// weights never meet non-finite values.
//
// Warps, bf16 caches: 0-1 softmax (query rows 0-63; TMEM lanes 0-63), 4
// producer, 5 MMA issue (one lane) and TMEM owner, 2, 3, 6, 7 converters;
// fp8 caches: 0-3 softmax, 4 producer, 5 MMA issue, 6-9 converters.  Every
// wait is bounded (SPATTN_DEV_WAIT_TIMEOUT).
#pragma once

#include "attention.cuh"
#include "attention_tc.cuh"
#include "tcgen05.cuh"

namespace spattn {

// 8 warps; warp w runs on SM sub-partition w % 4.  The softmax warps (0, 1)
// share sub-partitions 0 and 1 only with the producer and the MMA issuer;
// the converters (warps 2, 3, 6, 7) have sub-partitions 2 and 3 to
// themselves.  Two warps per sub-partition leave room for 255 registers.
constexpr int kTcwThreads = 8 * 32;           // bf16 caches
constexpr int kTcwThreadsFp8 = 10 * 32;       // fp8 caches
__host__ __device__ constexpr int tcw_threads(bool fp8) { return fp8 ? kTcwThreadsFp8 : kTcwThreads; }
constexpr int kTcwRows = 64;                  // query rows per unit, at most
constexpr int kTcwConvWarps = 4;
// Converter warps: bf16 caches 2, 3, 6, 7 (sub-partitions 2 and 3, beside the
// two softmax warps 0 and 1); fp8 caches 6, 7, 8, 9 (the softmax warps are
// 0-3 there).  0..3 for a converter warp, else -1.
template <bool FP8>
__device__ __forceinline__ int tcw_conv_index(int warp) {
    if (FP8) return warp >= 6 && warp < 10 ? warp - 6 : -1;
    return warp == 2 ? 0 : warp == 3 ? 1 : warp == 6 ? 2 : warp == 7 ? 3 : -1;
}
// Softmax warps and partial records per (CTA, unit) slot: bf16 caches two
// warps, one record; fp8 caches four warps in two halves (tokens 0-31 and
// 32-63 of a block, each with its own reference maximum), two records.
__host__ __device__ constexpr int tcw_softmax_warps(bool fp8) { return fp8 ? 4 : 2; }
__host__ __device__ constexpr int tcw_records(bool fp8) { return fp8 ? 2 : 1; }
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

// Shared memory: two query slots (64 rows x 128 bf16 as two 64-column halves,
// or the two e4m3 terms of the rows), kPB P buffers (128 rows x 64 bf16 or
// f16), the copy stages and operands below, then meta and barriers.  Operand
// tiles on 1024-byte boundaries.
//
// bf16 caches: kSrc = kOp stages, each the K and V operands of one block
// (copied straight into the operand layout), released when the block's PV
// product is done.
// fp8 caches: a ring of kSrc copy stages, each [K codes 8 KB | V codes 8
// KB] of one block (the K codes are the QK operand as copied), released once
// the block's QK product is done and its V codes are converted; and kOp = 3
// buffers of converted V (f16 operand), released by the PV product.  A copy
// stage therefore lives for the copy, QK and the conversion only, so that
// many blocks' copies are in flight.  Meta entries outlive the stage (the PV
// product reads them last): kMeta = kSrc + 8, see the producer.
template <bool FP8>
struct TcwLayout {
    static constexpr int kOp = FP8 ? 3 : 4;          // bf16: stages; fp8: converted V buffers
    static constexpr int kSrc = FP8 ? 4 : kOp;       // the ring the copies land in
    // P buffers (and their PV products): fp8 three, so that neither the
    // softmax (writing P) nor the converters (writing V) wait for the PV
    // product of the tile before the previous one
    static constexpr int kPB = FP8 ? 3 : 2;
    static constexpr int kMeta = FP8 ? kSrc + 8 : kOp;
    // bf16: 64 rows x 128 bf16; fp8: the two e4m3 terms, each 128 rows (the
    // 64 query rows twice, for the two softmax halves) x 128 bytes
    static constexpr int kQSlot = FP8 ? 2 * 128 * 128 : kTcwRows * 256;
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + 2 * kQSlot;                   // [kPB] P buffers
    static constexpr int kOffK = kOffP + kPB * 128 * 128;              // bf16: K operands; fp8: the copy ring
    static constexpr int kOffV = kOffK + kSrc * 16384;                 // V operands
    static constexpr int kOffMeta = kOffV + kOp * 16384;
    static constexpr int kNBars = 2 * kSrc + kOp + 2 * kPB + 4 * 2 + 2;
    static constexpr int kOffBars = align16(kOffMeta + kMeta * (int)sizeof(TcwMeta));
    static constexpr int kSmem = align16(kOffBars + kNBars * 8 + 16);
};

// Two e4m3 codes (low byte first) -> two f16 (low half first): one hardware
// conversion, exact (every e4m3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(codes & 0xffffu)));
    return h2;
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], 8-bit operands (32 elements of K per product).
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Two floats -> two e4m3 codes (x0 in the low byte), round to nearest even,
// saturating at +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float x0, float x1) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
    return r;
}

// f16 instruction descriptor (kind::f16 with f16 A and B), fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
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

// 32 consecutive 32-bit TMEM columns of this thread's lane, one load.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <bool FP8>
__global__ void __launch_bounds__(tcw_threads(FP8), 1)
    attn_tcw_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, AttnArgs a) {
    using TL = TcwLayout<FP8>;
    constexpr int kOp = TL::kOp, kSrc = TL::kSrc, kMeta = TL::kMeta, kPB = TL::kPB;
    static_assert(!FP8 || kOp == kPB, "fp8: V buffer of tile k is k % kPB, the PV buffers' index");
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *pbuf = smem + TL::kOffP;
    TcwMeta *meta = reinterpret_cast<TcwMeta *>(smem + TL::kOffMeta);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TL::kOffBars);
    uint64_t *full = bars;                      // [kSrc] copies landed
    uint64_t *empty = full + kSrc;              // [kSrc] the copy stage may be refilled
    uint64_t *conv = empty + kSrc;              // [kOp] bf16: stage's operands ready; fp8: V buffer converted
    // per-buffer barriers ([k & 1] for tile k), so that no parity wait can
    // be lapped by a phase two tiles ahead
    uint64_t *s_full = conv + kOp;              // [2] S buffer computed
    uint64_t *s_free = s_full + 2;              // [2] S buffer read (warps 0, 1)
    uint64_t *p_full = s_free + 2;              // [kPB] P buffer written, rescales done (softmax warps)
    uint64_t *pv_done = p_full + kPB;           // [kPB] the PV product of that buffer completed
    uint64_t *q_free = pv_done + kPB;           // [2] query slot's last product completed
    uint64_t *q_read = q_free + 2;              // [2] fp8: the slot's row scales read (warps 0, 1)
    uint64_t *fin = q_read + 2;                 // MMA issuer: all products completed
    uint64_t *done = fin + 1;                   // warps 0-3 finished with TMEM
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    // fp8 caches: the keys' codes straight from the copy, the query as two
    // e4m3 terms (two products into S); bf16: one bf16 product
    constexpr uint32_t kIdescQK = FP8 ? umma_idesc_e4m3(128, 64, false, false) : umma_idesc_bf16(128, 64, false, false);
    __shared__ float s_qinv[2][kTcwRows];   // fp8: 2^-e of each query row's scaling
    // fp8 caches: one f16 product (weights and values in f16); bf16: hi / lo
    constexpr uint32_t kIdescPV = FP8 ? umma_idesc_f16(128, 128, false, true) : umma_idesc_bf16(128, 128, false, true);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSrc; ++s) {
            mbar_init(&full[s], 1);
            // fp8: the QK product's commit and every converter warp
            mbar_init(&empty[s], FP8 ? 1 + kTcwConvWarps : 1);
        }
        for (int s = 0; s < kOp; ++s) mbar_init(&conv[s], kTcwConvWarps);
        for (int p = 0; p < 2; ++p) {
            mbar_init(&s_full[p], 1);
            mbar_init(&s_free[p], tcw_softmax_warps(FP8));
            mbar_init(&q_free[p], 1);
            mbar_init(&q_read[p], tcw_softmax_warps(FP8));
        }
        for (int p = 0; p < kPB; ++p) {
            mbar_init(&p_full[p], tcw_softmax_warps(FP8));
            mbar_init(&pv_done[p], 1);
        }
        mbar_init(fin, 1);
        mbar_init(done, tcw_softmax_warps(FP8));
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTcwTmemCols);
        tmem_relinquish();
    }
    if (FP8) {
        // the P halves a thread never writes stay zero
        for (int i = threadIdx.x; i < kPB * 16384 / 16; i += blockDim.x)
            reinterpret_cast<uint4 *>(pbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
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
        int i_push = 0, seg = -1;
        // Push one stage (whole warp, uniformly): wait for the stage, at a
        // segment start wait for the query slot and fill it, then lane 0
        // writes the stage's meta and issues the copies.
        auto push = [&](int unit, int j, int page, int flags, int nvalid) -> bool {
            // the stage is free once its products (bf16), or its QK product
            // and its conversion (fp8), are done.  (fp8: refilling stage s
            // with tile i needs the QK product of tile i - kSrc, which needs
            // the softmax to have read the scores of tile i - kSrc - 2; by
            // then the PV product of every tile before i - kSrc - 4 is done,
            // so meta entry i % kMeta, kMeta = kSrc + 8, is no longer read.)
            const int s = i_push % kSrc;
            int okw = 1;
            if (lane == 0 && i_push >= kSrc) okw = mbar_wait(&empty[s], ((i_push / kSrc) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
            int qs = seg & 1;
            if (flags & kFirst) {
                ++seg;
                qs = seg & 1;
                if (lane == 0 && seg >= 2) {
                    okw = mbar_wait(&q_free[qs], ((seg >> 1) - 1) & 1);
                    // fp8: the softmax warps took the slot's row scales of its
                    // previous segment (they read them at that segment's start)
                    if (FP8 && okw) okw = mbar_wait(&q_read[qs], ((seg >> 1) - 1) & 1);
                }
                if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
                // the segment's query rows, zero padded: bf16 as stored, or
                // (fp8 caches) each row scaled by 2^e (its largest element in
                // [2^7, 2^8)) and split into two e4m3 terms q1 + q2 (exact for
                // the elements within 2^9 of the row's largest), one 64-row
                // panel of 128-byte rows each
                // (row tile `tile` of the request and KV head's Tq * group rows)
                const int un = unit / a.ntiles, tile = unit % a.ntiles;
                const int b = un / a.hkv, h = un % a.hkv;
                uint8_t *qd = smem + TL::kOffQ + qs * TL::kQSlot;
                for (int task = lane; task < kTcwRows * 16; task += 32) {
                    const int row = task >> 4, c8 = task & 15;   // a half-warp holds one row
                    const int rg = tile * kTcwRows + row;         // the row in the whole chunk
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (row < a.rows && rg < a.rows_total) {
                        const int t = rg / a.group, g = rg % a.group;
                        v = *reinterpret_cast<const uint4 *>(
                            a.q + (((int64_t)b * a.tq + t) * a.hq + h * a.group + g) * kHeadDim + c8 * 8);
                    }
                    if (!FP8) {
                        *reinterpret_cast<uint4 *>(qd + qslot_offset(row, c8 * 8, kTcwRows)) = v;
                    } else {
                        float f[8];
                        bf16x8_to_f32(v, f);
                        float mx = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
#pragma unroll
                        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        // e = 7 - floor(log2 mx), kept inside the fp32 exponent range
                        int ex = mx > 0.f ? 7 - (int)((__float_as_uint(mx) >> 23) & 0xff) + 127 : 0;
                        ex = ex < -100 ? -100 : (ex > 100 ? 100 : ex);
                        const float sc = __uint_as_float((uint32_t)(ex + 127) << 23);   // 2^ex
                        uint32_t w1[4], w2[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x0 = f[2 * e] * sc, x1 = f[2 * e + 1] * sc;
                            w1[e] = f32x2_to_e4m3x2(x0, x1);
                            float h0, h1;   // the first term back in fp32 (exact)
                            e4m3x2_to_f32((uint16_t)w1[e], h0, h1);
                            w2[e] = f32x2_to_e4m3x2(x0 - h0, x1 - h1);
                        }
                        // 8 bytes at byte column c8 * 8 of the row (128-byte swizzle)
                        const int off = (row >> 3) * 1024 + (row & 7) * 128 + ((((c8 >> 1) ^ row) & 7) << 4) +
                                        (c8 & 1) * 8;
                        // the row twice (rows r and 64 + r: 8 KiB apart) in each
                        // term's 128-row panel (16 KiB apart)
                        const uint2 t1 = make_uint2(w1[0] | (w1[1] << 16), w1[2] | (w1[3] << 16));
                        const uint2 t2 = make_uint2(w2[0] | (w2[1] << 16), w2[2] | (w2[3] << 16));
                        *reinterpret_cast<uint2 *>(qd + off) = t1;
                        *reinterpret_cast<uint2 *>(qd + 8192 + off) = t1;
                        *reinterpret_cast<uint2 *>(qd + 16384 + off) = t2;
                        *reinterpret_cast<uint2 *>(qd + 16384 + 8192 + off) = t2;
                        if (c8 == 0) s_qinv[qs][row] = __uint_as_float((uint32_t)(127 - ex) << 23);   // 2^-ex
                    }
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                float ks = 1.f, vs = 1.f;
                const int h = (unit / a.ntiles) % a.hkv;
                if (FP8 && page >= 0) {
                    ks = a.k_scale[(int64_t)page * a.hkv + h];
                    vs = a.v_scale[(int64_t)page * a.hkv + h];
                }
                meta[i_push % kMeta] = TcwMeta{j, page, unit, flags, seg, nvalid, qs, ks, vs, {0, 0, 0}};
                if (page >= 0) {
                    const int y = (page * a.hkv + h) * kBlock;
                    if (FP8) {
                        mbar_arrive_expect_tx(&full[s], 2 * 8192);
                        tma_load_2d(smem + TL::kOffK + s * 16384, &kmap, 0, y, &full[s], kv_policy);   // codes: the operand
                        tma_load_2d(smem + TL::kOffK + s * 16384 + 8192, &vmap, 0, y, &full[s], kv_policy);
                    } else {
                        mbar_arrive_expect_tx(&full[s], 4 * 8192);
                        tma_load_2d(smem + TL::kOffK + s * 16384, &kmap, 0, y, &full[s], kv_policy);
                        tma_load_2d(smem + TL::kOffK + s * 16384 + 8192, &kmap, 64, y, &full[s], kv_policy);
                        tma_load_2d(smem + TL::kOffV + s * 16384, &vmap, 0, y, &full[s], kv_policy);
                        tma_load_2d(smem + TL::kOffV + s * 16384 + 8192, &vmap, 64, y, &full[s], kv_policy);
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
                const int b = unit / a.ntiles / a.hkv;
                const int ia = (int)(lo > us ? lo - us : 0);
                const int ib = (int)(hi - us < uc ? hi - us : uc);
                const int32_t *sel = a.sel_idx + (int64_t)(unit / a.ntiles) * a.max_sel;
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

    if (tcw_conv_index<FP8>(warp) >= 0) {
        // ========================================================== converters
        // Stage by stage: fp8 codes -> bf16 operand boxes, V rows of unfilled
        // slots zeroed; then the operands are released to the MMA issuer.
        // Lanes take consecutive tokens of one 16-column chunk: both the
        // 128-byte-swizzled staging rows and the operand rows are then read
        // and written without bank conflicts.
        const int ct = tcw_conv_index<FP8>(warp) * 32 + lane;   // 0 .. 32 * kTcwConvWarps - 1
        for (int i = 0;; ++i) {
            const int rs = i % kSrc, os = i % kOp;
            if (!mbar_wait(&full[rs], (i / kSrc) & 1)) break;
            const TcwMeta m = meta[i % kMeta];
            if (FP8 && (m.flags & kEnd)) break;
            // fp8: V buffer os is free once the PV product of tile i - kOp is done
            if (FP8 && i >= kOp && !mbar_wait(&pv_done[os], ((i / kOp) - 1) & 1)) break;
            if (m.page >= 0) {
                uint8_t *vop = smem + TL::kOffV + os * 16384;
                if (FP8) {
                    const uint8_t *stg = smem + TL::kOffK + rs * 16384;   // [K codes | V codes]
#pragma unroll
                    for (int e = 0; e < 512 / (kTcwConvWarps * 32); ++e) {
                        // V only (the K codes are the QK operand as copied)
                        const int task = ct + e * kTcwConvWarps * 32;
                        const int tt = task & 63, c16 = (task >> 6) & 7;   // token, 16-column chunk
                        const uint4 u = *reinterpret_cast<const uint4 *>(stg + 8192 + tt * 128 +
                                                                         ((c16 ^ (tt & 7)) << 4));
                        // to f16: the PV product takes f16 weights and values
                        uint4 w0 = make_uint4(e4m3x2_to_f16x2(u.x), e4m3x2_to_f16x2(u.x >> 16),
                                              e4m3x2_to_f16x2(u.y), e4m3x2_to_f16x2(u.y >> 16));
                        uint4 w1 = make_uint4(e4m3x2_to_f16x2(u.z), e4m3x2_to_f16x2(u.z >> 16),
                                              e4m3x2_to_f16x2(u.w), e4m3x2_to_f16x2(u.w >> 16));
                        if (tt >= m.nvalid) w0 = w1 = make_uint4(0u, 0u, 0u, 0u);
                        uint8_t *box = vop + (c16 >> 2) * 8192;
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
            if (lane == 0) {
                mbar_arrive(&conv[os]);
                if (FP8) mbar_arrive(&empty[rs]);   // the V codes are converted
            }
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
                if (pv < qk && mbar_test_wait(&p_full[pv % kPB], (pv / kPB) & 1) &&
                    (!FP8 || mbar_test_wait(&conv[pv % kOp], (pv / kOp) & 1))) {   // first: a PV product frees a stage
                    tc_fence_after();
                    const int s = pv % kSrc;
                    const TcwMeta m = meta[pv % kMeta];
                    if (m.page >= 0) {
                        const uint32_t acc0 = last_seg == m.seg ? 1u : 0u;
                        last_seg = m.seg;
                        const uint32_t vb = smem_u32(smem + TL::kOffV + (FP8 ? pv % kOp : s) * 16384);
                        const uint32_t pb = smem_u32(pbuf + (pv % kPB) * 16384);
                        // O hi += P rows 0-63 . V ; O lo += P rows 64-127 . V (the
                        // other 64 lanes of each product are never read)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t bd = sw128_desc(vb + ks * 2048, 8192, 1024);
                            umma_bf16(tbase + kTcwOHi, sw128_desc(pb + ks * 32, 16, 1024), bd, kIdescPV,
                                      ks > 0 ? 1u : acc0);
                            if (!FP8)
                                umma_bf16(tbase + kTcwOLo, sw128_desc(pb + 8192 + ks * 32, 16, 1024), bd, kIdescPV,
                                          ks > 0 ? 1u : acc0);
                        }
                        umma_commit(&pv_done[pv % kPB]);
                        if (!FP8) umma_commit(&empty[s]);
                    } else {
                        mbar_arrive(&pv_done[pv % kPB]);
                        if (!FP8) mbar_arrive(&empty[s]);
                    }
                    ++pv;
                    progressed = true;
                }
                if (qk < n) {
                    const int s = qk % kSrc, j = qk & 1;
                    // bf16: the stage's operands are ready; fp8: the copied K
                    // codes are the operand (the V conversion only gates PV)
                    if ((FP8 ? mbar_test_wait(&full[s], (qk / kSrc) & 1) : mbar_test_wait(&conv[s], (qk / kOp) & 1)) &&
                        (qk < 2 || mbar_test_wait(&s_free[j], ((qk >> 1) - 1) & 1))) {
                        const TcwMeta m = meta[qk % kMeta];
                        if (m.flags & kEnd) {
                            n = qk;
                            if (FP8) mbar_arrive(&s_full[j]);   // the softmax warps learn the end here
                        } else {
                            tc_fence_after();
                            if (m.page >= 0) {
                                const uint32_t qb = smem_u32(smem + TL::kOffQ + m.qslot * TL::kQSlot);
                                const uint32_t kb = smem_u32(smem + TL::kOffK + s * 16384);
                                if (FP8) {
                                    // S = q1 . K + q2 . K, 32 elements of d per product
#pragma unroll
                                    for (int ks = 0; ks < 8; ++ks) {
                                        const uint64_t ad = sw128_desc(qb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                                        const uint64_t bd = sw128_desc(kb + (ks & 3) * 32, 16, 1024);
                                        umma_f8(tbase + j * 64, ad, bd, kIdescQK, ks > 0);
                                    }
                                } else {
#pragma unroll
                                    for (int ks = 0; ks < 8; ++ks) {
                                        const uint64_t ad =
                                            sw128_desc(qb + (ks >> 2) * (kTcwRows * 128) + (ks & 3) * 32, 16, 1024);
                                        const uint64_t bd = sw128_desc(kb + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                                        umma_bf16(tbase + j * 64, ad, bd, kIdescQK, ks > 0);
                                    }
                                }
                                umma_commit(&s_full[j]);
                                if (FP8) umma_commit(&empty[s]);   // the K codes are no longer read
                            } else {
                                mbar_arrive(&s_full[j]);
                                if (FP8) mbar_arrive(&empty[s]);
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

    // ============================================== softmax (warps 0, 1; fp8: 0-3)
    // fp8: warps 2h, 2h + 1 take tokens 32h .. 32h + 31 of every block for
    // the 64 query rows (the query operand holds the rows twice, so TMEM lane
    // 64h + r holds row r's scores); each half keeps its own reference
    // maximum, sum and accumulator rows and writes its own partial record.
    const int half = FP8 ? warp >> 1 : 0;
    const int r = (FP8 ? (warp & 1) : warp) * 32 + lane;  // query row
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lane quarter
    constexpr int NT = FP8 ? 32 : 64;                     // a block's tokens per thread
    int t_r = 0;             // the row's chunk token (in the current segment's row tile)
    bool row_ok = false;     // the row exists in that tile

    constexpr float kSlack = FP8 ? 15.f : kTcSlack;   // f16 weights stay below 2^15
    float m_ref = -INFINITY, l_run = 0.f;
    float q_inv = 1.f;   // fp8: 2^-e, the scaling of this row's query in the current segment
    int cur_seg = -1, unit = 0, L = 0, k_last = -1;
    bool had_pv = false;
    // wait for tile kk's PV products (its buffer's barrier)
    auto wait_pv = [&](int kk) -> bool { return mbar_wait(&pv_done[kk % kPB], (kk / kPB) & 1); };
    auto rescale_o = [&](float f) {   // both parts of this row's accumulator
#pragma unroll 1
        for (int cc = 0; cc < (FP8 ? 8 : 16); ++cc) {
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
        // bf16: the operands of tile k are ready (which publishes its meta);
        // fp8: its scores are (the MMA issuer read the meta first)
        if (!mbar_wait(FP8 ? &s_full[k & 1] : &conv[k % kOp], FP8 ? (k >> 1) & 1 : (k / kOp) & 1)) break;
        const TcwMeta md = meta[k % kMeta];
        const bool end = md.flags & kEnd;
        if (cur_seg >= 0 && (end || md.seg != cur_seg)) {
            // ---- end of a segment: this row's partial record (m, l, O = hi + lo)
            if (k_last >= 0 && !wait_pv(k_last)) break;
            tc_fence_after();
            const int64_t rec = (((int64_t)c + unit) * tcw_records(FP8) + half) * a.rows + r;
            const uint64_t keep = l2_evict_last();   // the merge reads the record next
            if (row_ok) st_global_f2(a.part_ml + rec * 2, m_ref, l_run, keep);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                float v[16], w[16];
                if (had_pv) {
                    tmem_ld16(tbase + lanes + kTcwOHi + cc * 16, v);
                    if (!FP8) {
                        tmem_ld16(tbase + lanes + kTcwOLo + cc * 16, w);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] += w[e];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0.f;
                }
                if (row_ok) {
                    float *dst = a.part_o + rec * kHeadDim + cc * 16;
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
            L = a.seq_lens[unit / a.ntiles / a.hkv];
            L = (L < 0 || L > a.max_blocks * kBlock) ? 0 : L;
            {
                const int rg = (unit % a.ntiles) * kTcwRows + r;
                row_ok = r < a.rows && rg < a.rows_total;
                t_r = rg / a.group;
            }
            had_pv = false;
            m_ref = -INFINITY;
            l_run = 0.f;
            if (FP8) {
                // this row's query scale for the segment; the slot may then be refilled
                q_inv = s_qinv[md.qslot][r];
                __syncwarp();
                if (lane == 0) mbar_arrive(&q_read[md.qslot]);
            }
        }
        const bool valid = md.page >= 0;
        const int j = k & 1;
        // ---- this row's 64 scores (one TMEM load), log2 units, masked
        if (!FP8 && !mbar_wait(&s_full[j], (k >> 1) & 1)) break;
        tc_fence_after();
        float x[NT];
        if (valid) {
            if constexpr (FP8)
                tmem_ld32(tbase + lanes + j * 64 + half * 32, x);
            else
                tmem_ld64(tbase + lanes + j * 64, x);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[j]);
        float alpha = 1.f;
        uint32_t hw[NT / 2], lw[NT / 2];
        if (valid) {
            const int lim = min(L - 1, L - a.tq + t_r);   // last position the row sees
            const float sc = FP8 ? a.qscale * md.ks * q_inv : a.qscale * md.ks;
            const int pos0 = md.j * kBlock + half * 32;
            float mx = -INFINITY;
            if (row_ok && pos0 + NT - 1 <= lim) {   // all of this thread's tokens are visible to the row
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    x[t] *= sc;
                    mx = fmaxf(mx, x[t]);
                }
            } else {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    x[t] = (row_ok && pos0 + t <= lim) ? x[t] * sc : -INFINITY;
                    mx = fmaxf(mx, x[t]);
                }
            }
            // the weights enter P times the block's V scale, 2^(x + log2 vs - m):
            // the reference m follows x + log2 vs, so that every weight stays
            // below 2^slack (f16 weights for fp8 caches: below 2^15 < 65504);
            // the row sum takes 2^(x - m), the weights divided by the scale
            const float lvs = md.vs == 1.f ? 0.f : __log2f(md.vs);
            const float my = mx + lvs;
            if (my > m_ref + kSlack || (m_ref == -INFINITY && mx != -INFINITY)) {
                alpha = m_ref == -INFINITY ? 0.f : exp2f(m_ref - my);
                m_ref = my;
                l_run *= alpha;
            }
            const float mu = (m_ref == -INFINITY ? 0.f : m_ref) - lvs;
            float ps = 0.f;
#pragma unroll
            for (int e = 0; e < NT / 2; ++e) {
                const float p0 = ex2_ftz(x[2 * e] - mu), p1 = ex2_ftz(x[2 * e + 1] - mu);
                ps += p0 + p1;
                if (FP8) {
                    // one f16 weight (11 significant bits)
                    const __half2 h = __floats2half2_rn(p0, p1);
                    hw[e] = *reinterpret_cast<const uint32_t *>(&h);
                } else {
                    // hi = p with its low 16 bits cleared (a bf16 value), lo =
                    // the exact fp32 remainder, truncated the same way: the
                    // pair keeps ~15 significant bits, with integer ops only
                    // (the exp2 pipe stays free for the exponentials)
                    const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
                    const float r0 = p0 - __uint_as_float(b0 & 0xffff0000u);
                    const float r1 = p1 - __uint_as_float(b1 & 0xffff0000u);
                    hw[e] = __byte_perm(b0, b1, 0x7632);
                    lw[e] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
                }
            }
            l_run += md.vs == 1.f ? ps : ps / md.vs;
        }
        const float a_o = (valid && had_pv) ? alpha : 1.f;
        // ---- P buffer k % kPB is free once tile k - kPB's products are done
        const int jp = k % kPB;
        if (k >= kPB && !wait_pv(k - kPB)) break;
        if (valid) {
            if (a_o != 1.f) {
                // rescale this row's accumulator: after tile k - 1's products
                if (k >= 1 && !wait_pv(k - 1)) break;
                tc_fence_after();
                rescale_o(a_o);
            }
            uint8_t *pb = pbuf + jp * 16384;
            if constexpr (FP8) {
                // P row 64h + r, tokens 32h .. 32h + 31; the other half of the
                // row stays zero (cleared at the start, never written)
                const int prow = warp * 32 + lane;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(pb + sw128_offset(prow, half * 32 + c8 * 8)) =
                        make_uint4(hw[4 * c8], hw[4 * c8 + 1], hw[4 * c8 + 2], hw[4 * c8 + 3]);
            } else {
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    *reinterpret_cast<uint4 *>(pb + sw128_offset(r, c8 * 8)) =
                        make_uint4(hw[4 * c8], hw[4 * c8 + 1], hw[4 * c8 + 2], hw[4 * c8 + 3]);
                    *reinterpret_cast<uint4 *>(pb + sw128_offset(64 + r, c8 * 8)) =
                        make_uint4(lw[4 * c8], lw[4 * c8 + 1], lw[4 * c8 + 2], lw[4 * c8 + 3]);
                }
            }
            fence_proxy_async_smem();
            had_pv = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[jp]);
        k_last = k;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(done);
}

}  // namespace spattn
