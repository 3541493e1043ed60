// spattn.cu -- C ABI of libspattn: argument checks, workspace layout and
// kernel launches.  Every kernel lives in the headers included below; this
// is the only translation unit, so the device status word is one symbol.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <utility>

#include "spattn.h"
#include "common.cuh"
#include "compress.cuh"
#include "scores.cuh"
#include "select.cuh"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "attention_tcw.cuh"
#include "merge.cuh"
#include "hca.cuh"

using namespace spattn;

namespace {

thread_local std::string g_err;

spattn_status fail(spattn_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

spattn_status ok() {
    g_err.clear();
    return SPATTN_OK;
}

#define SP_TRY(expr)                                  \
    do {                                              \
        spattn_status _st = (expr);                   \
        if (_st != SPATTN_OK) return _st;             \
    } while (0)

spattn_status cuda_ok(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return SPATTN_OK;
    return fail(SPATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Upper bound on persistent attention CTAs (one per SM, for devices of up to
// 320 SMs); the workspace is sized for it so that workspace sizes need no
// device query.
constexpr int kMaxAttnCtas = 2 * 160;
constexpr int kMaxRows = 4096;   // query rows per (request, KV head): Tq * Hq / Hkv
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool pow2_hkv(int h) { return h == 1 || h == 2 || h == 4 || h == 8 || h == 16; }

spattn_status check_dims(const spattn_dims *d) {
    if (!d) return fail(SPATTN_ERR_INVALID_ARG, "dims is NULL");
    if (d->batch < 1 || d->q_tokens < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 ||
        d->num_pages < 1 || d->max_blocks_per_seq < 1 || d->max_sel < 0)
        return fail(SPATTN_ERR_INVALID_ARG, "dims: sizes must be positive");
    if (d->head_dim != kHeadDim)
        return fail(SPATTN_ERR_UNSUPPORTED, "head_dim %d: only %d is built", d->head_dim, kHeadDim);
    if (d->block_size != kBlock)
        return fail(SPATTN_ERR_UNSUPPORTED, "block_size %d: only %d is built", d->block_size, kBlock);
    if (d->num_q_heads % d->num_kv_heads)
        return fail(SPATTN_ERR_INVALID_ARG, "num_q_heads %d is not a multiple of num_kv_heads %d",
                    d->num_q_heads, d->num_kv_heads);
    if (!pow2_hkv(d->num_kv_heads))
        return fail(SPATTN_ERR_UNSUPPORTED, "num_kv_heads %d: built for 1, 2, 4, 8, 16", d->num_kv_heads);
    if (d->kbar_dtype != SPATTN_KBAR_F32 && d->kbar_dtype != SPATTN_KBAR_BF16)
        return fail(SPATTN_ERR_INVALID_ARG, "kbar_dtype %d", d->kbar_dtype);
    const int64_t rows = (int64_t)d->q_tokens * (d->num_q_heads / d->num_kv_heads);
    if (rows > kMaxRows)
        return fail(SPATTN_ERR_UNSUPPORTED, "q_tokens * num_q_heads / num_kv_heads = %lld > %d",
                    (long long)rows, kMaxRows);
    if (d->kv_dtype != SPATTN_KV_BF16 && d->kv_dtype != SPATTN_KV_FP8_E4M3)
        return fail(SPATTN_ERR_INVALID_ARG, "kv_dtype %d", d->kv_dtype);
    if ((int64_t)d->max_blocks_per_seq * kBlock > INT32_MAX / 2)
        return fail(SPATTN_ERR_UNSUPPORTED, "max_blocks_per_seq too large");
    return SPATTN_OK;
}

spattn_status check_params(const spattn_params *p) {
    if (!p) return fail(SPATTN_ERR_INVALID_ARG, "params is NULL");
    if (p->sink_blocks < 0 || p->local_blocks < 0)
        return fail(SPATTN_ERR_INVALID_ARG, "sink_blocks and local_blocks must be >= 0");
    if (p->mode != SPATTN_SEL_TOPK && p->mode != SPATTN_SEL_TOPP && p->mode != SPATTN_SEL_TOPP_ANCHOR)
        return fail(SPATTN_ERR_INVALID_ARG, "mode %d", p->mode);
    if (p->top_k < 0) return fail(SPATTN_ERR_INVALID_ARG, "top_k %d < 0", p->top_k);
    if (p->mode != SPATTN_SEL_TOPK && !(p->top_p > 0.f && p->top_p <= 1.f))
        return fail(SPATTN_ERR_INVALID_ARG, "top_p %g not in (0, 1]", (double)p->top_p);
    if (!(p->max_ratio >= 0.f && p->max_ratio <= 1.f))
        return fail(SPATTN_ERR_INVALID_ARG, "max_ratio %g not in [0, 1]", (double)p->max_ratio);
    if (!(p->sm_scale >= 0.f) || !std::isfinite(p->sm_scale))
        return fail(SPATTN_ERR_INVALID_ARG, "sm_scale %g", (double)p->sm_scale);
    if (p->mode == SPATTN_SEL_TOPP_ANCHOR &&
        !(p->max_ratio > 0.f && p->min_ratio >= 0.f && p->min_ratio <= p->max_ratio))
        return fail(SPATTN_ERR_INVALID_ARG, "anchor mode needs 0 <= min_ratio (%g) <= max_ratio (%g), max_ratio > 0",
                    (double)p->min_ratio, (double)p->max_ratio);
    return SPATTN_OK;
}

int n_mid_cap(const spattn_dims *d, const spattn_params *p) {
    const int64_t n = (int64_t)d->max_blocks_per_seq - p->sink_blocks - p->local_blocks;
    return n > 0 ? (int)n : 0;
}

int k_max_of(const spattn_params *p, int n_mid) {
    if (p->max_ratio > 0.f) {
        const int k = (int)std::floor((double)p->max_ratio * (double)n_mid);
        return k < n_mid ? k : n_mid;
    }
    return n_mid;
}

int32_t required_max_sel(const spattn_dims *d, const spattn_params *p) {
    const int nm = n_mid_cap(d, p);
    const int km = k_max_of(p, nm);
    int k = km;
    if (p->mode == SPATTN_SEL_TOPK && p->top_k > 0 && p->top_k < k) k = p->top_k;
    const int64_t mid = std::min<int64_t>(nm, (int64_t)d->q_tokens * k);
    const int64_t req = (int64_t)p->sink_blocks + p->local_blocks + mid;
    return (int32_t)std::min<int64_t>(req, d->max_blocks_per_seq);
}

float sm_scale_of(const spattn_params *p) {
    return p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt((float)kHeadDim);
}

int rows_of(const spattn_dims *d) { return d->q_tokens * (d->num_q_heads / d->num_kv_heads); }
// Row tiles of (at most) 64 query rows per (request, KV head) for the
// attention, and the rows of one tile (the stride of the partial records).
int row_tiles(const spattn_dims *d) { return (rows_of(d) + kTcwRows - 1) / kTcwRows; }
int tile_rows(const spattn_dims *d) { return std::min(rows_of(d), kTcwRows); }

// Attention runs on the tensor cores: attn_tc_kernel for bf16 caches with
// at most kTcNQ query rows per KV head, attn_tcw_kernel for the rest (fp8
// caches, or up to kTcwRows rows).
bool uses_tc(const spattn_dims *d) { return d->kv_dtype == SPATTN_KV_BF16 && rows_of(d) <= kTcNQ; }

// Partial records per (CTA, unit) slot: one per softmax warp (attn_tc), one
// (attn_tcw).
int records_per_slot(const spattn_dims *d) {
    return uses_tc(d) ? kTcWarpSlots : tcw_records(d->kv_dtype == SPATTN_KV_FP8_E4M3);
}

// Per-device caches (SM count; which kernels have their shared-memory limit
// raised).  Guarded by one mutex: these are host-side set-up calls only.
std::mutex g_mu;
std::map<std::pair<int, const void *>, int> g_smem_set;

// Raise a kernel's dynamic shared-memory limit (per device and kernel) to
// the largest size asked for so far, so that a call needing more than an
// earlier one raises it again.
spattn_status ensure_smem(const void *func, int bytes) {
    if (bytes <= 48 * 1024) return SPATTN_OK;
    int dev;
    SP_TRY(cuda_ok(cudaGetDevice(&dev), "cudaGetDevice"));
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_smem_set.find({dev, func});
    if (it != g_smem_set.end() && it->second >= bytes) return SPATTN_OK;
    SP_TRY(cuda_ok(cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                   "cudaFuncSetAttribute"));
    g_smem_set[{dev, func}] = bytes;
    return SPATTN_OK;
}

std::map<int, int> g_sms;

// SM count of the current device, queried once per device (so that calls
// captured into a CUDA graph after the first one make no attribute query).
spattn_status sm_count(int *out) {
    int dev;
    SP_TRY(cuda_ok(cudaGetDevice(&dev), "cudaGetDevice"));
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) {
        *out = it->second;
        return SPATTN_OK;
    }
    SP_TRY(cuda_ok(cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev),
                   "cudaDeviceGetAttribute"));
    g_sms[dev] = *out;
    return SPATTN_OK;
}

constexpr int kMaxSmem = 227 * 1024;

struct DecodeLayout {
    size_t scores_off, scores_bytes, part_o_off, part_ml_off, total;
};

// Workspace: [scores] | partial outputs | partial (max, sum).  (C_max +
// units) slots of `rows` query rows, records_per_slot() records per slot;
// units count every 64-row tile of a (request, KV head) separately.  The
// scores are there for spattn_decode without scores_out.
DecodeLayout decode_layout(const spattn_dims *d, bool with_scores) {
    DecodeLayout L{};
    const int64_t units = (int64_t)d->batch * d->num_kv_heads * row_tiles(d);
    const int64_t slots = (kMaxAttnCtas + units) * records_per_slot(d);
    const int64_t rows = tile_rows(d);
    size_t off = 0;
    L.scores_off = off;
    L.scores_bytes = with_scores ? align_up((size_t)d->batch * d->q_tokens * d->num_kv_heads *
                                            d->max_blocks_per_seq * sizeof(float))
                                 : 0;
    off += L.scores_bytes;
    L.part_o_off = off;
    off += align_up((size_t)(slots * rows) * kHeadDim * sizeof(float));
    L.part_ml_off = off;
    off += align_up((size_t)(slots * rows) * 2 * sizeof(float));
    L.total = off;
    return L;
}

// ------------------------------------------------------------- launches

// Plain stream-ordered launch through cudaLaunchKernelEx.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch whose CTAs may be scheduled before the previous kernel in the
// stream has finished (programmatic dependent launch): the kernel runs its
// input-independent prologue, then waits (griddepcontrol.wait) for the
// previous grid's completion and memory before reading its results.
template <typename... KArgs, typename... Args>
cudaError_t launch_early(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args &&...args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

spattn_status launch_scores(const spattn_dims *d, const spattn_params *p, const void *q,
                            const void *kbar, const int32_t *bt, const int32_t *sl, float *scores,
                            cudaStream_t st) {
    ScoresArgs a;
    a.q = static_cast<const uint16_t *>(q);
    a.kbar = kbar;
    a.block_table = bt;
    a.seq_lens = sl;
    a.scores = scores;
    a.tq = d->q_tokens;
    a.hq = d->num_q_heads;
    a.num_pages = d->num_pages;
    a.max_blocks = d->max_blocks_per_seq;
    a.sink = p->sink_blocks;
    a.local = p->local_blocks;
    a.anchors = p->mode == SPATTN_SEL_TOPP_ANCHOR;
    a.scale = sm_scale_of(p);
    // query tokens per CTA: at most 128 (token, KV head) rows of q-bar
    a.tt = std::max(1, std::min(d->q_tokens, 128 / d->num_kv_heads));
    const int rowsq = a.tt * d->num_kv_heads;
    const int ztiles = (d->q_tokens + a.tt - 1) / a.tt;
    // (with 8 KV heads a one-wave grid of more blocks per CTA measured slower;
    // with one or two, faster: score_blocks_per_cta)
    const int bpc_min = score_blocks_per_cta(rowsq);
    auto smem_of = [&](int bpc) {
        return rowsq * (kHeadDim + bpc) * (int)sizeof(float) + bpc * (int)sizeof(int);
    };
    if (smem_of(bpc_min) > kMaxSmem)
        return fail(SPATTN_ERR_UNSUPPORTED, "q_tokens * num_kv_heads = %d too large for block scores", rowsq);
    const bool kb16 = d->kbar_dtype == SPATTN_KBAR_BF16;
    const void *fn = nullptr;
#define SP_SCORES_FN(H) (kb16 ? (const void *)block_scores_kernel<H, true> : (const void *)block_scores_kernel<H, false>)
    switch (d->num_kv_heads) {
        case 1: fn = SP_SCORES_FN(1); break;
        case 2: fn = SP_SCORES_FN(2); break;
        case 4: fn = SP_SCORES_FN(4); break;
        case 8: fn = SP_SCORES_FN(8); break;
        case 16: fn = SP_SCORES_FN(16); break;
    }
#undef SP_SCORES_FN
    a.bpc = bpc_min;
    const int smem = smem_of(a.bpc);
    dim3 grid((d->max_blocks_per_seq + a.bpc - 1) / a.bpc, d->batch, ztiles);
    SP_TRY(ensure_smem(fn, smem));
    cudaError_t e = cudaSuccess;
#define SP_SCORES_LAUNCH(H)                                                                     \
    e = kb16 ? launch(block_scores_kernel<H, true>, grid, kScoreThreads, smem, st, a)          \
             : launch(block_scores_kernel<H, false>, grid, kScoreThreads, smem, st, a)
    switch (d->num_kv_heads) {
        case 1: SP_SCORES_LAUNCH(1); break;
        case 2: SP_SCORES_LAUNCH(2); break;
        case 4: SP_SCORES_LAUNCH(4); break;
        case 8: SP_SCORES_LAUNCH(8); break;
        case 16: SP_SCORES_LAUNCH(16); break;
    }
#undef SP_SCORES_LAUNCH
    return cuda_ok(e, "block_scores launch");
}

// The selection is launched early (programmatic dependent launch): its CTAs
// may start while the kernel before it in the stream finishes, and wait for
// it before reading anything that kernel may write.  `behind_scores`: the
// kernel before it is block_scores_kernel of the same decode call, so the
// request lengths (which it does not write) may be read before the wait.
spattn_status launch_select(const spattn_dims *d, const spattn_params *p, const float *scores,
                            const int32_t *sl, int32_t *sel_idx, int32_t *sel_count, bool behind_scores,
                            cudaStream_t st) {
    SelectArgs a;
    a.scores = scores;
    a.seq_lens = sl;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.tq = d->q_tokens;
    a.hkv = d->num_kv_heads;
    a.max_blocks = d->max_blocks_per_seq;
    a.max_sel = d->max_sel;
    a.sink = p->sink_blocks;
    a.local = p->local_blocks;
    a.mode = p->mode;
    a.min_ratio = p->min_ratio;
    a.top_k = p->top_k;
    a.top_p = p->top_p;
    a.max_ratio = p->max_ratio;
    a.n_mid_cap = std::max(1, n_mid_cap(d, p));
    a.len_early = behind_scores ? 1 : 0;
    a.sort_cap = 0;
    if (p->mode != SPATTN_SEL_TOPK) {
        const int km = std::max(1, k_max_of(p, n_mid_cap(d, p)));
        int np2 = 1;
        while (np2 < km) np2 <<= 1;
        a.sort_cap = np2;
    }
    const size_t smem = select_smem_bytes(a.n_mid_cap, a.sort_cap, a.max_blocks);
    if (smem > (size_t)kMaxSmem)
        return fail(SPATTN_ERR_UNSUPPORTED, "selection needs %zu bytes of shared memory (max_blocks %d)",
                    smem, a.max_blocks);
    // latency-bound: the fewest threads that still cover a row in a few
    // passes (measured: 512 beat 1024 by 15-25 % on 2K-4K middle blocks)
    const int nm = n_mid_cap(d, p);
    const int threads = nm <= 1024 ? 256 : (nm <= 4096 ? 512 : kSelThreads);
    const unsigned rows = (unsigned)(d->batch * d->num_kv_heads);
    SP_TRY(ensure_smem((const void *)select_kernel, (int)smem));
    return cuda_ok(launch_early(select_kernel, dim3(rows), dim3(threads), smem, st, a), "select launch");
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// 2-D view of a bf16 cache as [num_pages * Hkv * 64 token rows][128], boxes
// of 64 x 64 with 128-byte swizzle (the tensor-core operand layout).
spattn_status kv_tensor_map_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        SP_TRY(cuda_ok(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q),
                       "cudaGetDriverEntryPoint"));
        if (!fn || q != cudaDriverEntryPointSuccess)
            return fail(SPATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return SPATTN_OK;
}

spattn_status kv_tensor_map(CUtensorMap *m, const void *base, int64_t rows) {
    SP_TRY(kv_tensor_map_encoder());
    const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SPATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SPATTN_OK;
}

// 2-D view of an fp8 cache as [num_pages * Hkv * 64 token rows][128 bytes],
// boxes of one whole (page, head) tile (64 rows x 128 bytes), 128-byte
// swizzle (the staging buffer the converter warps read).
spattn_status kv_tensor_map_u8(CUtensorMap *m, const void *base, int64_t rows) {
    SP_TRY(kv_tensor_map_encoder());
    const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim};
    const cuuint32_t box[2] = {128, 64};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SPATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SPATTN_OK;
}

// Tensor-core path for many rows and fp8 caches: one CTA per SM.
template <bool FP8>
spattn_status launch_attn_tcw(AttnArgs &a, const void *k_cache, const void *v_cache, int sms, cudaStream_t st,
                              int *ctas_out) {
    CUtensorMap kmap, vmap;
    const int64_t rows = (int64_t)a.num_pages * a.hkv * kBlock;
    if (FP8) {
        SP_TRY(kv_tensor_map_u8(&kmap, k_cache, rows));
        SP_TRY(kv_tensor_map_u8(&vmap, v_cache, rows));
    } else {
        SP_TRY(kv_tensor_map(&kmap, k_cache, rows));
        SP_TRY(kv_tensor_map(&vmap, v_cache, rows));
    }
    const int smem = TcwLayout<FP8>::kSmem;
    SP_TRY(ensure_smem((const void *)attn_tcw_kernel<FP8>, smem));
    const int ctas = std::min(kMaxAttnCtas, sms);
    *ctas_out = ctas;
    return cuda_ok(launch_early(attn_tcw_kernel<FP8>, dim3(ctas), dim3(tcw_threads(FP8)), smem, st, kmap, vmap, a),
                   "attention (tensor core, many rows) launch");
}

// Tensor-core path: bf16 caches, at most kTcNQ query rows per KV head.  One
// CTA per SM (all of its TMEM), rows rounded up to 4, 8 or 16.
template <int RQ>
spattn_status launch_attn_tc_t(AttnArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap, int sms,
                               cudaStream_t st, int *ctas_out) {
    const int smem = TcLayout<RQ>::kSmem;
    const void *fn = (const void *)attn_tc_kernel<RQ>;
    SP_TRY(ensure_smem(fn, smem));
    const int ctas = std::min(kMaxAttnCtas, sms);
    *ctas_out = ctas;
    return cuda_ok(launch_early(attn_tc_kernel<RQ>, dim3(ctas), dim3(kTcThreads), smem, st, kmap, vmap, a),
                   "attention (tensor core) launch");
}

spattn_status launch_attn_tc(AttnArgs &a, const void *k_cache, const void *v_cache, int sms, cudaStream_t st,
                             int *ctas_out) {
    CUtensorMap kmap, vmap;
    const int64_t rows = (int64_t)a.num_pages * a.hkv * kBlock;
    SP_TRY(kv_tensor_map(&kmap, k_cache, rows));
    SP_TRY(kv_tensor_map(&vmap, v_cache, rows));
    if (a.rows <= 4) return launch_attn_tc_t<4>(a, kmap, vmap, sms, st, ctas_out);
    if (a.rows <= 8) return launch_attn_tc_t<8>(a, kmap, vmap, sms, st, ctas_out);
    return launch_attn_tc_t<16>(a, kmap, vmap, sms, st, ctas_out);
}

spattn_status launch_attention(const spattn_dims *d, const spattn_params *p, const void *q,
                               const void *k_cache, const void *v_cache, const float *k_scale,
                               const float *v_scale, const int32_t *bt, const int32_t *sl,
                               const int32_t *sel_idx, const int32_t *sel_count, float *out,
                               float *lse, char *ws, const DecodeLayout &L, cudaStream_t st) {
    const bool fp8 = d->kv_dtype == SPATTN_KV_FP8_E4M3;
    const int rows = rows_of(d);
    int sms;
    SP_TRY(sm_count(&sms));
    AttnArgs a;
    a.q = static_cast<const uint16_t *>(q);
    a.k_cache = static_cast<const uint8_t *>(k_cache);
    a.v_cache = static_cast<const uint8_t *>(v_cache);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.block_table = bt;
    a.seq_lens = sl;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.part_o = reinterpret_cast<float *>(ws + L.part_o_off);
    a.part_ml = reinterpret_cast<float *>(ws + L.part_ml_off);
    a.tq = d->q_tokens;
    a.hq = d->num_q_heads;
    a.hkv = d->num_kv_heads;
    a.group = d->num_q_heads / d->num_kv_heads;
    a.rows = tile_rows(d);
    a.rows_total = rows;
    a.ntiles = row_tiles(d);
    a.units = d->batch * d->num_kv_heads * a.ntiles;
    a.num_pages = d->num_pages;
    a.max_blocks = d->max_blocks_per_seq;
    a.max_sel = d->max_sel;
    a.qscale = sm_scale_of(p) * kLog2e;
    const bool tc = uses_tc(d);
    int ctas = 0;
    if (tc)
        SP_TRY(launch_attn_tc(a, k_cache, v_cache, sms, st, &ctas));
    else
        SP_TRY(fp8 ? launch_attn_tcw<true>(a, k_cache, v_cache, sms, st, &ctas)
                   : launch_attn_tcw<false>(a, k_cache, v_cache, sms, st, &ctas));

    MergeArgs m;
    m.part_o = a.part_o;
    m.part_ml = a.part_ml;
    m.sel_count = sel_count;
    m.out = out;
    m.lse = lse;
    m.batch = d->batch;
    m.tq = d->q_tokens;
    m.hq = d->num_q_heads;
    m.hkv = d->num_kv_heads;
    m.group = a.group;
    m.rows = a.rows;
    m.units = a.units;
    m.ntiles = a.ntiles;
    m.max_sel = d->max_sel;
    m.ctas = ctas;
    m.wslots = records_per_slot(d);
    m.pairs = tc ? 1 : 0;
    // one CTA per output row; warps for the records a unit gets on average
    // (CTAs per unit + 1, times the records per CTA), a group of 16 or 20 per warp
    const int64_t nrows = (int64_t)d->batch * d->q_tokens * d->num_q_heads;
    const int64_t recs = ((int64_t)ctas / std::max(1, a.units) + 2) * m.wslots;
    int wpr = 1;
    while (wpr < kMergeMaxWarps && merge_group(wpr) * wpr < recs) wpr *= 2;
    const dim3 grid((unsigned)nrows), block(32 * wpr);
    cudaError_t e;
    switch (wpr) {
        case 1: e = launch_early(merge_kernel<1>, grid, block, 0, st, m); break;
        case 2: e = launch_early(merge_kernel<2>, grid, block, 0, st, m); break;
        case 4: e = launch_early(merge_kernel<4>, grid, block, 0, st, m); break;
        case 8: e = launch_early(merge_kernel<8>, grid, block, 0, st, m); break;
        default: e = launch_early(merge_kernel<16>, grid, block, 0, st, m); break;
    }
    return cuda_ok(e, "merge launch");
}

spattn_status check_cache_args(const spattn_dims *d, const void *q, const void *k_cache,
                               const void *v_cache, const float *k_scale, const float *v_scale,
                               const int32_t *bt, const int32_t *sl) {
    if (!q || !k_cache || !v_cache || !bt || !sl)
        return fail(SPATTN_ERR_INVALID_ARG, "q, k_cache, v_cache, block_table, seq_lens are required");
    if (d->kv_dtype == SPATTN_KV_FP8_E4M3 && (!k_scale || !v_scale))
        return fail(SPATTN_ERR_INVALID_ARG, "fp8 caches need k_scale and v_scale");
    if (((uintptr_t)k_cache | (uintptr_t)v_cache) & 15)
        return fail(SPATTN_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
    if ((uintptr_t)q & 15) return fail(SPATTN_ERR_INVALID_ARG, "q must be 16-byte aligned");
    return SPATTN_OK;
}

// ------------------------------------------------ fixed scratch (no allocation)

// Scratch of spattn_decode_selected_noalloc: a module-scope device array, one
// instance on every device that loads this library, held until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::map<int, void *> g_noalloc_ptr;

// Device address of the scratch array on the current device.  In host code
// the array's name is only a stand-in, so the address is asked for once per
// device (with that device current) and cached.
spattn_status noalloc_scratch(void **out) {
    int dev;
    SP_TRY(cuda_ok(cudaGetDevice(&dev), "cudaGetDevice"));
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_noalloc_ptr.find(dev);
    if (it != g_noalloc_ptr.end()) {
        *out = it->second;
        return SPATTN_OK;
    }
    void *p = nullptr;
    SP_TRY(cuda_ok(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)"));
    g_noalloc_ptr[dev] = p;
    *out = p;
    return SPATTN_OK;
}

template <int RQ>
constexpr bool tc_layout_ok() {
    using TL = TcLayout<RQ>;
    return TL::kSmem <= 227 * 1024 && TL::kStages % 2 == 0 && TL::kOffQ % 1024 == 0 && TL::kQSlot % 1024 == 0 &&
           TL::kOffP % 1024 == 0 && TL::kOffRing % 1024 == 0 && kTcBox % 1024 == 0 && TL::kOffP >= TL::kOffQ + 1024;
}
static_assert(tc_layout_ok<4>() && tc_layout_ok<8>() && tc_layout_ok<16>(),
              "one CTA per SM; even stage count; swizzled operand tiles on 1024-byte boundaries");
template <bool FP8>
constexpr bool tcw_layout_ok() {
    using TL = TcwLayout<FP8>;
    return TL::kSmem <= 227 * 1024 && TL::kOffP % 1024 == 0 && TL::kOffK % 1024 == 0 && TL::kOffV % 1024 == 0 &&
           TL::kOffMeta % 16 == 0 && TL::kOffQ % 1024 == 0;
}
static_assert(tcw_layout_ok<false>() && tcw_layout_ok<true>(), "many-row tensor-core layout");

// Split of the HCA attention: CTAs per (request, KV head), so that all
// CTAs fit in one wave at two per SM.
int hca_split(int units, int sms) {
    const int s = 2 * sms / units;
    return s < 1 ? 1 : (s > kHcaMaxSplit ? kHcaMaxSplit : s);
}

size_t hca_workspace_bytes(const spattn_dims *d) {
    const size_t recs = (size_t)d->batch * d->num_kv_heads * kHcaMaxSplit * rows_of(d);
    return align_up(recs * kHeadDim * 4) + align_up(recs * 2 * 4);
}

// The HCA branch's attention (optionally merged with another branch's
// result): partial records per share of the entries, then their merge.
spattn_status launch_hca_attend(const spattn_dims *d, const spattn_params *p, const void *q, const float *khat,
                                const float *vhat, const int32_t *sl, const float *base_out,
                                const float *base_lse, float *out, float *lse, void *workspace,
                                size_t workspace_bytes, cudaStream_t st) {
    SP_TRY(check_dims(d));
    SP_TRY(check_params(p));
    if (!q || !khat || !vhat || !sl || !out)
        return fail(SPATTN_ERR_INVALID_ARG, "q, khat, vhat, seq_lens, out are required");
    if (((uintptr_t)q | (uintptr_t)khat | (uintptr_t)vhat | (uintptr_t)out) & 15)
        return fail(SPATTN_ERR_INVALID_ARG, "q, khat, vhat and out must be 16-byte aligned");
    const size_t need = hca_workspace_bytes(d);
    if (!workspace || workspace_bytes < need)
        return fail(SPATTN_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", workspace_bytes, need);
    if ((uintptr_t)workspace & (kAlign - 1))
        return fail(SPATTN_ERR_WORKSPACE, "workspace must be %zu-byte aligned", kAlign);
    int sms;
    SP_TRY(sm_count(&sms));
    const int units = d->batch * d->num_kv_heads;
    const size_t recs = (size_t)units * kHcaMaxSplit * rows_of(d);
    HcaAttendArgs a;
    a.q = static_cast<const uint16_t *>(q);
    a.khat = khat;
    a.vhat = vhat;
    a.seq_lens = sl;
    a.part_o = static_cast<float *>(workspace);
    a.part_ml = reinterpret_cast<float *>(static_cast<char *>(workspace) + align_up(recs * kHeadDim * 4));
    a.tq = d->q_tokens;
    a.hq = d->num_q_heads;
    a.hkv = d->num_kv_heads;
    a.max_blocks = d->max_blocks_per_seq;
    a.gmax = (d->max_blocks_per_seq + kHcaGroupBlocks - 1) / kHcaGroupBlocks;
    a.split = hca_split(units, sms);
    a.qscale = sm_scale_of(p) * kLog2e;
    const dim3 grid(a.split, units), block(32 * (kHcaCtaWarps + 1));
    cudaError_t e;
    if (rows_of(d) <= 4) {
        SP_TRY(ensure_smem((const void *)hca_partial_kernel<4, 8>, HcaRing<8>::kSmem));
        e = launch(hca_partial_kernel<4, 8>, grid, block, HcaRing<8>::kSmem, st, a);
    } else {
        SP_TRY(ensure_smem((const void *)hca_partial_kernel<8, 4>, HcaRing<4>::kSmem));
        e = launch(hca_partial_kernel<8, 4>, grid, block, HcaRing<4>::kSmem, st, a);
    }
    SP_TRY(cuda_ok(e, "hca_partial launch"));
    HcaCombineArgs c;
    c.part_o = a.part_o;
    c.part_ml = a.part_ml;
    c.base_out = base_out;
    c.base_lse = base_lse;
    c.out = out;
    c.lse = lse;
    c.nrows = (int64_t)d->batch * d->q_tokens * d->num_q_heads;
    c.tq = d->q_tokens;
    c.hq = d->num_q_heads;
    c.hkv = d->num_kv_heads;
    c.split = a.split;
    SP_TRY(cuda_ok(launch(hca_combine_kernel, dim3((unsigned)((c.nrows + 7) / 8)), dim3(256), 0, st, c),
                   "hca_combine launch"));
    return ok();
}

}  // namespace

// ================================================================ C ABI

extern "C" {

int32_t spattn_required_max_sel(const spattn_dims *dims, const spattn_params *params) {
    if (check_dims(dims) != SPATTN_OK || check_params(params) != SPATTN_OK) return -1;
    return required_max_sel(dims, params);
}

spattn_status spattn_compress_keys(const spattn_dims *dims, const void *k_cache, const float *k_scale,
                                   const int32_t *block_table, const int32_t *old_lens,
                                   const int32_t *seq_lens, void *kbar, spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    if (!k_cache || !block_table || !seq_lens || !kbar)
        return fail(SPATTN_ERR_INVALID_ARG, "k_cache, block_table, seq_lens, kbar are required");
    const bool fp8 = dims->kv_dtype == SPATTN_KV_FP8_E4M3;
    if (fp8 && !k_scale) return fail(SPATTN_ERR_INVALID_ARG, "fp8 caches need k_scale");
    if (((uintptr_t)k_cache & 15) || ((uintptr_t)kbar & 15))
        return fail(SPATTN_ERR_INVALID_ARG, "k_cache and kbar must be 16-byte aligned");
    CompressArgs a;
    a.k_cache = static_cast<const uint8_t *>(k_cache);
    a.k_scale = k_scale;
    a.block_table = block_table;
    a.old_lens = old_lens;
    a.seq_lens = seq_lens;
    a.kbar = kbar;
    a.kbar_bf16 = dims->kbar_dtype == SPATTN_KBAR_BF16;
    a.hkv = dims->num_kv_heads;
    a.num_pages = dims->num_pages;
    a.max_blocks = dims->max_blocks_per_seq;
    const int gx = old_lens ? (dims->q_tokens + kBlock - 1) / kBlock + 1 : dims->max_blocks_per_seq;
    dim3 grid(gx, dims->batch);
    const int tg = compress_groups(dims->num_kv_heads);
    const int threads = tg * dims->num_kv_heads * 16;
    const int smem = threads * 2 * (int)sizeof(float4);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define SP_COMPRESS(F, T) compress_keys_kernel<F, T><<<grid, threads, smem, st>>>(a)
    if (fp8) {
        if (tg == 8) SP_COMPRESS(true, 8); else if (tg == 4) SP_COMPRESS(true, 4); else SP_COMPRESS(true, 2);
    } else {
        if (tg == 8) SP_COMPRESS(false, 8); else if (tg == 4) SP_COMPRESS(false, 4); else SP_COMPRESS(false, 2);
    }
#undef SP_COMPRESS
    SP_TRY(cuda_ok(cudaGetLastError(), "compress_keys launch"));
    return ok();
}

spattn_status spattn_block_scores(const spattn_dims *dims, const spattn_params *params, const void *q,
                                  const void *kbar, const int32_t *block_table,
                                  const int32_t *seq_lens, float *scores, spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    SP_TRY(check_params(params));
    if (!q || !kbar || !block_table || !seq_lens || !scores)
        return fail(SPATTN_ERR_INVALID_ARG, "q, kbar, block_table, seq_lens, scores are required");
    if (((uintptr_t)kbar & 15)) return fail(SPATTN_ERR_INVALID_ARG, "kbar must be 16-byte aligned");
    SP_TRY(launch_scores(dims, params, q, kbar, block_table, seq_lens, scores,
                         reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

spattn_status spattn_select(const spattn_dims *dims, const spattn_params *params, const float *scores,
                            const int32_t *seq_lens, int32_t *sel_idx, int32_t *sel_count,
                            spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    SP_TRY(check_params(params));
    if (!scores || !seq_lens || !sel_idx || !sel_count)
        return fail(SPATTN_ERR_INVALID_ARG, "scores, seq_lens, sel_idx, sel_count are required");
    const int32_t need = required_max_sel(dims, params);
    if (dims->max_sel < need)
        return fail(SPATTN_ERR_INVALID_ARG, "max_sel %d < required %d", dims->max_sel, need);
    SP_TRY(launch_select(dims, params, scores, seq_lens, sel_idx, sel_count, false,
                         reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

size_t spattn_decode_workspace_size(const spattn_dims *dims, const spattn_params *params) {
    if (check_dims(dims) != SPATTN_OK || check_params(params) != SPATTN_OK) return 0;
    return decode_layout(dims, true).total;
}

spattn_status spattn_decode_selected(const spattn_dims *dims, const spattn_params *params, const void *q,
                                     const void *k_cache, const void *v_cache, const float *k_scale,
                                     const float *v_scale, const int32_t *block_table,
                                     const int32_t *seq_lens, const int32_t *sel_idx,
                                     const int32_t *sel_count, float *out, void *workspace,
                                     size_t workspace_bytes, spattn_stream_t stream) {
    return spattn_decode_selected_lse(dims, params, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                                      sel_idx, sel_count, out, nullptr, workspace, workspace_bytes, stream);
}

spattn_status spattn_decode_selected_lse(const spattn_dims *dims, const spattn_params *params, const void *q,
                                         const void *k_cache, const void *v_cache, const float *k_scale,
                                         const float *v_scale, const int32_t *block_table,
                                         const int32_t *seq_lens, const int32_t *sel_idx,
                                         const int32_t *sel_count, float *out, float *lse, void *workspace,
                                         size_t workspace_bytes, spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    SP_TRY(check_params(params));
    SP_TRY(check_cache_args(dims, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens));
    if (!sel_idx || !sel_count || !out)
        return fail(SPATTN_ERR_INVALID_ARG, "sel_idx, sel_count, out are required");
    if ((uintptr_t)out & 15) return fail(SPATTN_ERR_INVALID_ARG, "out must be 16-byte aligned");
    const DecodeLayout L = decode_layout(dims, false);
    if (!workspace || workspace_bytes < L.total)
        return fail(SPATTN_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", workspace_bytes, L.total);
    if ((uintptr_t)workspace & (kAlign - 1))
        return fail(SPATTN_ERR_WORKSPACE, "workspace must be %zu-byte aligned", kAlign);
    char *ws = static_cast<char *>(workspace);
    SP_TRY(launch_attention(dims, params, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                            sel_idx, sel_count, out, lse, ws, L, reinterpret_cast<cudaStream_t>(stream)));
    return ok();
}

spattn_status spattn_decode_selected_noalloc(const spattn_dims *dims, const spattn_params *params,
                                             const void *q, const void *k_cache, const void *v_cache,
                                             const float *k_scale, const float *v_scale,
                                             const int32_t *block_table, const int32_t *seq_lens,
                                             const int32_t *sel_idx, const int32_t *sel_count, float *out,
                                             spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    SP_TRY(check_params(params));
    SP_TRY(check_cache_args(dims, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens));
    if (!sel_idx || !sel_count || !out)
        return fail(SPATTN_ERR_INVALID_ARG, "sel_idx, sel_count, out are required");
    if ((uintptr_t)out & 15) return fail(SPATTN_ERR_INVALID_ARG, "out must be 16-byte aligned");
    const DecodeLayout L = decode_layout(dims, false);
    if (L.total > kNoAllocScratchBytes)
        return fail(SPATTN_ERR_UNSUPPORTED,
                    "these dims need %zu bytes of scratch; the built-in scratch holds %zu bytes "
                    "(use spattn_decode_selected with a workspace)",
                    L.total, kNoAllocScratchBytes);
    void *scratch = nullptr;
    SP_TRY(noalloc_scratch(&scratch));
    char *ws = static_cast<char *>(scratch);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    SP_TRY(launch_attention(dims, params, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                            sel_idx, sel_count, out, nullptr, ws, L, st));
    return ok();
}

spattn_status spattn_decode(const spattn_dims *dims, const spattn_params *params, const void *q,
                            const void *k_cache, const void *v_cache, const float *k_scale,
                            const float *v_scale, const int32_t *block_table, const int32_t *seq_lens,
                            const void *kbar, float *out, int32_t *sel_idx, int32_t *sel_count,
                            float *scores_out, void *workspace, size_t workspace_bytes,
                            spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    SP_TRY(check_params(params));
    SP_TRY(check_cache_args(dims, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens));
    if (!kbar || !out || !sel_idx || !sel_count)
        return fail(SPATTN_ERR_INVALID_ARG, "kbar, out, sel_idx, sel_count are required");
    if (((uintptr_t)kbar | (uintptr_t)out) & 15)
        return fail(SPATTN_ERR_INVALID_ARG, "kbar and out must be 16-byte aligned");
    const int32_t need = required_max_sel(dims, params);
    if (dims->max_sel < need)
        return fail(SPATTN_ERR_INVALID_ARG, "max_sel %d < required %d", dims->max_sel, need);
    const DecodeLayout L = decode_layout(dims, scores_out == nullptr);
    if (!workspace || workspace_bytes < L.total)
        return fail(SPATTN_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", workspace_bytes, L.total);
    if ((uintptr_t)workspace & (kAlign - 1))
        return fail(SPATTN_ERR_WORKSPACE, "workspace must be %zu-byte aligned", kAlign);
    char *ws = static_cast<char *>(workspace);
    float *scores = scores_out ? scores_out : reinterpret_cast<float *>(ws + L.scores_off);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    SP_TRY(launch_scores(dims, params, q, kbar, block_table, seq_lens, scores, st));
    SP_TRY(launch_select(dims, params, scores, seq_lens, sel_idx, sel_count, true, st));
    SP_TRY(launch_attention(dims, params, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                            sel_idx, sel_count, out, nullptr, ws, L, st));
    return ok();
}

// ---------------------------------------------------------------- HCA branch

int32_t spattn_hca_entries(const spattn_dims *dims) {
    if (check_dims(dims) != SPATTN_OK) return -1;
    return (dims->max_blocks_per_seq + kHcaGroupBlocks - 1) / kHcaGroupBlocks;
}

spattn_status spattn_hca_pool(const spattn_dims *dims, const void *k_cache, const void *v_cache,
                              const float *k_scale, const float *v_scale, const int32_t *block_table,
                              const int32_t *old_lens, const int32_t *seq_lens, float *khat, float *vhat,
                              spattn_stream_t stream) {
    SP_TRY(check_dims(dims));
    if (!k_cache || !v_cache || !block_table || !seq_lens || !khat || !vhat)
        return fail(SPATTN_ERR_INVALID_ARG, "k_cache, v_cache, block_table, seq_lens, khat, vhat are required");
    const bool fp8 = dims->kv_dtype == SPATTN_KV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return fail(SPATTN_ERR_INVALID_ARG, "fp8 caches need k_scale and v_scale");
    if (((uintptr_t)k_cache | (uintptr_t)v_cache | (uintptr_t)khat | (uintptr_t)vhat) & 15)
        return fail(SPATTN_ERR_INVALID_ARG, "k_cache, v_cache, khat and vhat must be 16-byte aligned");
    HcaPoolArgs a;
    a.k_cache = static_cast<const uint8_t *>(k_cache);
    a.v_cache = static_cast<const uint8_t *>(v_cache);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.block_table = block_table;
    a.old_lens = old_lens;
    a.seq_lens = seq_lens;
    a.khat = khat;
    a.vhat = vhat;
    a.hkv = dims->num_kv_heads;
    a.num_pages = dims->num_pages;
    a.max_blocks = dims->max_blocks_per_seq;
    a.gmax = spattn_hca_entries(dims);
    // incremental: the entries of the appended tokens (q_tokens of them, the
    // CTAs stride over more if a request grew further)
    const int gx = old_lens ? (dims->q_tokens + kHcaTokens - 1) / kHcaTokens + 1 : a.gmax;
    const dim3 grid(gx, dims->batch), block(kHcaPoolThreads);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (fp8)
        hca_pool_kernel<true><<<grid, block, 0, st>>>(a);
    else
        hca_pool_kernel<false><<<grid, block, 0, st>>>(a);
    SP_TRY(cuda_ok(cudaGetLastError(), "hca_pool launch"));
    return ok();
}

size_t spattn_hca_workspace_size(const spattn_dims *dims) {
    if (check_dims(dims) != SPATTN_OK) return 0;
    return hca_workspace_bytes(dims);
}

spattn_status spattn_hca_attend(const spattn_dims *dims, const spattn_params *params, const void *q,
                                const float *khat, const float *vhat, const int32_t *seq_lens, float *out,
                                float *lse, void *workspace, size_t workspace_bytes, spattn_stream_t stream) {
    if (!lse) return fail(SPATTN_ERR_INVALID_ARG, "lse is required");
    return launch_hca_attend(dims, params, q, khat, vhat, seq_lens, nullptr, nullptr, out, lse, workspace,
                             workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

spattn_status spattn_hca_attend_merge(const spattn_dims *dims, const spattn_params *params, const void *q,
                                      const float *khat, const float *vhat, const int32_t *seq_lens,
                                      const float *out_other, const float *lse_other, float *out, float *lse,
                                      void *workspace, size_t workspace_bytes, spattn_stream_t stream) {
    if (!out_other || !lse_other) return fail(SPATTN_ERR_INVALID_ARG, "out_other and lse_other are required");
    if ((uintptr_t)out_other & 15) return fail(SPATTN_ERR_INVALID_ARG, "out_other must be 16-byte aligned");
    return launch_hca_attend(dims, params, q, khat, vhat, seq_lens, out_other, lse_other, out, lse, workspace,
                             workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

spattn_status spattn_lse_merge(const spattn_dims *dims, const float *out_a, const float *lse_a,
                               const float *out_b, const float *lse_b, float *out, float *lse,
                               spattn_stream_t stream) {
    // only the row count and d matter here
    if (!dims) return fail(SPATTN_ERR_INVALID_ARG, "dims is NULL");
    if (dims->batch < 1 || dims->q_tokens < 1 || dims->num_q_heads < 1)
        return fail(SPATTN_ERR_INVALID_ARG, "dims: batch, q_tokens, num_q_heads must be positive");
    if (dims->head_dim != kHeadDim)
        return fail(SPATTN_ERR_UNSUPPORTED, "head_dim %d: only %d is built", dims->head_dim, kHeadDim);
    if (!out_a || !lse_a || !out_b || !lse_b || !out)
        return fail(SPATTN_ERR_INVALID_ARG, "out_a, lse_a, out_b, lse_b, out are required");
    if (((uintptr_t)out_a | (uintptr_t)out_b | (uintptr_t)out) & 15)
        return fail(SPATTN_ERR_INVALID_ARG, "out_a, out_b and out must be 16-byte aligned");
    const int64_t rows = (int64_t)dims->batch * dims->q_tokens * dims->num_q_heads;
    SP_TRY(cuda_ok(launch(lse_merge_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0,
                          reinterpret_cast<cudaStream_t>(stream), rows, out_a, lse_a, out_b, lse_b, out, lse),
                   "lse_merge launch"));
    return ok();
}

const char *spattn_last_error(void) { return g_err.c_str(); }

spattn_status spattn_get_device_status(int32_t *host_out, spattn_stream_t stream) {
    if (!host_out) return fail(SPATTN_ERR_INVALID_ARG, "host_out is NULL");
    SP_TRY(cuda_ok(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "cudaStreamSynchronize"));
    int32_t v = 0;
    SP_TRY(cuda_ok(cudaMemcpyFromSymbol(&v, g_status, sizeof v), "read status word"));
    const int32_t zero = 0;
    SP_TRY(cuda_ok(cudaMemcpyToSymbol(g_status, &zero, sizeof zero), "clear status word"));
    *host_out = v;
    return ok();
}

const char *spattn_version(void) { return "spattn 0.1 sm_100a"; }

}  // extern "C"
