/*
 * spattn.h -- C ABI of libspattn: block-sparse decode attention over a paged
 * KV cache, for NVIDIA B200 (sm_100a).
 *
 * For every query the library keeps the attention-sink block and the local
 * window blocks, scores the middle 64-token blocks against mean-pooled
 * (compressed) keys, keeps the best middle blocks by top-k or top-p, and runs
 * exact softmax attention over the kept blocks only.
 *
 * Sources of the operation (page titles as printed):
 *   "Claude Opus 长上下文 KV Cache 稀疏注意力", §稀疏注意力与 KV Cache 压缩的工程实现
 *     (block-level management, attention sink, local window, Top-P
 *     selection of middle blocks) and the configuration table of
 *     §可落地的配置参数与监控要点 (64-token blocks, 1 sink block, 2 local
 *     blocks, 10-20 % retention);
 *   "CSA + HCA 混合注意力机制", §4.1 (compress m tokens into one entry; plain
 *     averaging as the parameter-free compressor), §4.2 (score every
 *     compressed entry, top-k, attend over the selected entries only), §4.3
 *     (window + uncompressed tail join the attention), §4.4 (block-sparse
 *     pattern: score, select, softmax(q K_sel^T / sqrt(d)) V_sel), §2.3 (the
 *     decode step appends K, V then reads them back; the read is the
 *     bottleneck);
 *   "Claude Code压缩上下文窗口的底层原理与性能优化实践", 算法流程 (mean-pooling merge);
 *   "Claude Code 1M 上下文" (aicoding.csdn.net), §2(3) (FP8 KV storage).
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers into memory the caller owns, unless
 *     stated otherwise.  The library allocates nothing; scratch memory is the
 *     caller's `workspace`.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and never synchronises, except
 *     spattn_get_device_status.
 *   - Arguments are validated on the host before anything is enqueued; a bad
 *     argument returns SPATTN_ERR_INVALID_ARG (or _UNSUPPORTED) and enqueues
 *     nothing.  spattn_last_error() then describes it.
 *   - Bad DATA found on the device (a block-table entry outside
 *     [0, num_pages), a selected block past the request's end, a selection
 *     longer than max_sel, a bounded wait that gave up) never traps: the
 *     kernel skips the offending access, sets a bit in the device status
 *     word, and the result is unspecified.  Read and clear the word with
 *     spattn_get_device_status.
 *   - No C++ exception crosses this interface.
 *
 * Layouts (row-major, innermost last):
 *   q          bf16  [B][Tq][Hq][d]        query tokens; token t of request b
 *                                         sits at position seq_lens[b]-Tq+t
 *   k_cache    bf16 or fp8-e4m3fn bytes [num_pages][Hkv][P][d]   (HND pages)
 *   v_cache    same as k_cache
 *   k_scale    f32   [num_pages][Hkv]      fp8 only: value = code * scale
 *   v_scale    f32   [num_pages][Hkv]
 *   block_table int32 [B][max_blocks_per_seq]  logical block j -> page id
 *   seq_lens   int32 [B]                   tokens in the cache, including
 *                                         the Tq query tokens
 *   kbar       f32 or bf16 (dims.kbar_dtype) [num_pages][Hkv][d]
 *                                         mean-pooled key of each page
 *   scores     f32   [B][Tq][Hkv][max_blocks_per_seq]
 *   sel_idx    int32 [B][Hkv][max_sel]     kept logical block ids, ascending
 *   sel_count  int32 [B][Hkv]
 *   out        f32   [B][Tq][Hq][d]
 * Query head i reads KV head i / (Hq / Hkv).  d must be 128 and P must be 64.
 */
#ifndef SPATTN_H
#define SPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *spattn_stream_t;

typedef enum {
    SPATTN_OK = 0,
    SPATTN_ERR_INVALID_ARG = 1,   /* bad pointer, size or parameter */
    SPATTN_ERR_UNSUPPORTED = 2,   /* valid but not built (d != 128, P != 64, ...) */
    SPATTN_ERR_CUDA = 3,          /* a CUDA runtime call failed */
    SPATTN_ERR_WORKSPACE = 4,     /* workspace missing or too small */
    SPATTN_ERR_TIMEOUT = 5,       /* reserved for host-side waits */
    SPATTN_ERR_DEVICE = 6         /* the device status word is non-zero */
} spattn_status;

/* Bits of the device status word. */
#define SPATTN_DEV_BAD_PAGE      0x1   /* block-table entry outside [0, num_pages) */
#define SPATTN_DEV_BAD_BLOCK     0x2   /* selected block id outside [0, nb) */
#define SPATTN_DEV_SEL_OVERFLOW  0x4   /* a selection did not fit in max_sel */
#define SPATTN_DEV_WAIT_TIMEOUT  0x8   /* a bounded pipeline wait gave up */
#define SPATTN_DEV_BAD_LEN       0x10  /* seq_len < 0 or > max_blocks_per_seq * P */

typedef enum { SPATTN_KV_BF16 = 0, SPATTN_KV_FP8_E4M3 = 1 } spattn_kv_dtype;
/*
 * Storage of the compressed keys.  SPATTN_KBAR_BF16 halves the bytes the
 * block scores read: the fp32 mean rounded to bf16 (nearest even), scores
 * still accumulated in fp32 -- low-precision scoring after "CSA + HCA 混合注意力
 * 机制" §4.2 (the indexer's QK path runs at low precision; the page reports
 * 99.7 % top-k recall against BF16 for its FP4 path).
 */
typedef enum { SPATTN_KBAR_F32 = 0, SPATTN_KBAR_BF16 = 1 } spattn_kbar_dtype;
/*
 * Selection modes.  SPATTN_SEL_TOPP_ANCHOR: top-p whose retention cap adapts
 * to the anchors ("Claude Opus 长上下文 KV Cache 稀疏注意力", §多上下文场景下的跨文档
 * 注意力恢复, anchor-based dynamic selection: the sink and local blocks are
 * the anchors; the bounds (max, min) of the scores set the Top-P ratio, more
 * when the maximum stands well above the anchors, less otherwise).  Reading
 * taken (the page gives no formula): with a = the anchors' highest score and
 * hi / lo the middle blocks' highest / lowest score of the query row,
 * r = clamp((hi - a) / (hi - lo), 0, 1) (0 when hi <= lo), ratio = min_ratio
 * + r * (max_ratio - min_ratio), k_max = floor(ratio * n_mid) (computed in
 * double from the fp32 scores), then top-p with that cap.  block_scores then
 * scores the anchor blocks too (so the local blocks' compressed keys must be
 * current before it runs).
 */
typedef enum { SPATTN_SEL_TOPK = 0, SPATTN_SEL_TOPP = 1, SPATTN_SEL_TOPP_ANCHOR = 2 } spattn_sel_mode;

typedef struct {
    int32_t batch;              /* B >= 1 */
    int32_t q_tokens;           /* Tq >= 1: query tokens per request (1 = decode) */
    int32_t num_q_heads;        /* Hq, a multiple of Hkv; Tq * Hq / Hkv <= 4096 */
    int32_t num_kv_heads;       /* Hkv: 1, 2, 4, 8 or 16 */
    int32_t head_dim;           /* d, must be 128 */
    int32_t block_size;         /* P, must be 64 */
    int32_t num_pages;          /* pages in the cache pool (>= 1) */
    int32_t max_blocks_per_seq; /* columns of block_table and scores */
    int32_t max_sel;            /* columns of sel_idx; >= spattn_required_max_sel() */
    int32_t kv_dtype;           /* spattn_kv_dtype */
    int32_t kbar_dtype;         /* spattn_kbar_dtype of kbar */
} spattn_dims;

typedef struct {
    int32_t sink_blocks;        /* S >= 0: blocks [0, S) are always kept */
    int32_t local_blocks;       /* W >= 0: the last W blocks are always kept */
    int32_t mode;               /* spattn_sel_mode */
    int32_t top_k;              /* top-k: k when > 0, else k = k_max */
    float top_p;                /* top-p: mass threshold in (0, 1] */
    float max_ratio;            /* cap k_max = floor(max_ratio * n_mid), in
                                   [0, 1]; 0 means no cap (k_max = n_mid) */
    float sm_scale;             /* softmax and score scale; 0 = 1/sqrt(d) */
    float min_ratio;            /* SPATTN_SEL_TOPP_ANCHOR: ratio when the anchors
                                   dominate, in [0, max_ratio] (other modes ignore it) */
} spattn_params;

/*
 * Middle blocks of a request of nb = ceil(L / P) blocks are [S, nb - W);
 * n_mid = max(0, nb - S - W).  Per query token the kept middle set is
 *   top-k: the k = min(top_k > 0 ? top_k : k_max, k_max) best blocks, ranked
 *          by score descending, equal scores by lower block id;
 *   top-p: the shortest prefix of that ranking whose softmax probability
 *          (softmax over the middle blocks' scores) reaches top_p, cut to
 *          k_max blocks.
 * The kept set of (b, h) is sink + local + the union over the Tq tokens.
 */

/* Columns sel_idx needs for these dims and parameters:
 * min(max_blocks, S + W + min(n_mid, Tq * k)) at the longest request, with k
 * the largest per-token middle count the parameters allow.  Returns -1 on
 * invalid arguments. */
int32_t spattn_required_max_sel(const spattn_dims *dims, const spattn_params *params);

/*
 * spattn_compress_keys -- mean-pooled key of each block.
 * ("Claude Code压缩上下文窗口的底层原理与性能优化实践", 算法流程, 均值池化合并;
 *  "CSA + HCA 混合注意力机制" §4.1.)
 *
 * kbar[page][h][:] = mean over the filled tokens of block j of K (dequantised
 * with k_scale for fp8), for page = block_table[b][j], in fp32.  A block
 * holds min(P, L - j*P) tokens.  With old_lens == NULL every block of every
 * request is recomputed; otherwise only the blocks that hold a token of
 * [old_lens[b], seq_lens[b]) (the tokens appended since the last call).
 * k_scale may be NULL for bf16 caches.  Pages not touched keep their value.
 */
spattn_status spattn_compress_keys(const spattn_dims *dims, const void *k_cache,
                                   const float *k_scale, const int32_t *block_table,
                                   const int32_t *old_lens, const int32_t *seq_lens,
                                   void *kbar, spattn_stream_t stream);

/*
 * spattn_block_scores -- score every middle block.
 * ("CSA + HCA 混合注意力机制" §4.2 Lightning Indexer steps 3-4 and §4.4 step 1.)
 *
 * scores[b][t][h][j] = sm_scale * (qbar . kbar[block_table[b][j]][h]) for
 * middle blocks j, where qbar is the fp32 mean of the Hq/Hkv query rows of
 * token t that share KV head h; -inf in every other column (sink, local,
 * past the end).  fp32 arithmetic throughout.
 */
spattn_status spattn_block_scores(const spattn_dims *dims, const spattn_params *params,
                                  const void *q, const void *kbar,
                                  const int32_t *block_table, const int32_t *seq_lens,
                                  float *scores, spattn_stream_t stream);

/*
 * spattn_select -- sink + local + top-k / top-p middle blocks per (b, h).
 * ("Claude Opus 长上下文 KV Cache 稀疏注意力", §稀疏注意力与 KV Cache 压缩的工程实现;
 *  "CSA + HCA 混合注意力机制" §4.4 step 3.)
 *
 * Reads scores as written by spattn_block_scores (only the middle columns
 * are read) and writes the ascending kept block ids of (b, h) to
 * sel_idx[b][h][0 .. sel_count[b][h]).  Top-p probabilities and their running
 * sum are fp32.  Launched with programmatic dependent launch: the kernel
 * waits for the kernel before it in the stream to complete before it reads
 * any argument's memory (the scores, the lengths), so inputs written by
 * that kernel are seen.
 */
spattn_status spattn_select(const spattn_dims *dims, const spattn_params *params,
                            const float *scores, const int32_t *seq_lens,
                            int32_t *sel_idx, int32_t *sel_count, spattn_stream_t stream);

/* Bytes of workspace spattn_decode / spattn_decode_selected need (split-KV
 * partial results and, for spattn_decode without scores_out, the scores).
 * Returns 0 on invalid arguments. */
size_t spattn_decode_workspace_size(const spattn_dims *dims, const spattn_params *params);

/*
 * spattn_decode_selected -- exact attention over a given selection.
 * ("CSA + HCA 混合注意力机制" §2.1 and §4.4 step 4: softmax(q K_sel^T/sqrt(d)) V_sel.)
 *
 * out[b][t][i][:] = sum over tokens tau of the kept blocks of (b, h = i/G)
 * with position tau < seq_lens[b] and tau <= seq_lens[b] - Tq + t of
 * softmax_tau(sm_scale * q . k_tau) * v_tau, in fp32 (bf16 or fp8 inputs,
 * fp32 accumulation; split-KV partials merged by their log-sum-exp).
 * A row with no visible token is all zeros.  sel_idx / sel_count as written
 * by spattn_select (any ascending or unordered list of distinct ids works).
 * Both kernels run on the tensor cores (tcgen05): bf16 caches with
 * Tq * Hq / Hkv <= 16 with the tokens of a block on M (probabilities
 * entered as bf16 hi + lo parts); fp8 caches and larger row counts with the
 * query rows on M, in 64-row tiles (fp8: the scores from the key codes as
 * stored and the query split into two exact e4m3 terms, the values widened
 * e4m3 -> f16 exactly and weighted in f16; the scales applied to the scores
 * and the weights).  The kernels are launched with programmatic dependent
 * launch: each waits for the kernel before it in the stream to complete
 * before it reads any argument's memory, so inputs written by that kernel
 * are seen.
 */
spattn_status spattn_decode_selected(const spattn_dims *dims, const spattn_params *params,
                                     const void *q, const void *k_cache, const void *v_cache,
                                     const float *k_scale, const float *v_scale,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     const int32_t *sel_idx, const int32_t *sel_count,
                                     float *out, void *workspace, size_t workspace_bytes,
                                     spattn_stream_t stream);

/*
 * spattn_decode_selected_lse -- spattn_decode_selected that also reports each
 * row's log-sum-exp, so that its result can be combined with another
 * branch's over a disjoint key set ("CSA + HCA 混合注意力机制" §6: the sparse
 * and the compressed branches joined into one softmax).
 *
 * lse (device, fp32 [B][Tq][Hq], may be NULL = spattn_decode_selected)
 * receives ln(sum over the row's visible kept tokens of
 * exp(sm_scale * q . k_tau)), -inf for a row with no visible token.
 * Everything else as spattn_decode_selected.
 */
spattn_status spattn_decode_selected_lse(const spattn_dims *dims, const spattn_params *params,
                                         const void *q, const void *k_cache, const void *v_cache,
                                         const float *k_scale, const float *v_scale,
                                         const int32_t *block_table, const int32_t *seq_lens,
                                         const int32_t *sel_idx, const int32_t *sel_count,
                                         float *out, float *lse, void *workspace,
                                         size_t workspace_bytes, spattn_stream_t stream);

/*
 * spattn_decode_selected_noalloc -- spattn_decode_selected without a
 * caller-supplied workspace.  (Not a step of the method: the pages have no
 * counterpart; it only changes where the scratch memory lives.)
 *
 * For callers that cannot allocate device memory at the point of the call:
 * code running inside a host framework that owns every device allocation
 * (an engine plugin, a caching allocator that must not be bypassed), code
 * between the start and end of a CUDA stream capture, or latency-critical
 * loops that must not pay for an allocation or for the implicit device
 * synchronisation of freeing one.  The split-KV partial results go to a
 * fixed scratch array built into the library (16 MiB, a module-scope device
 * array present on every GPU that loads the library until the process
 * exits).  Arguments, layouts and results are those of
 * spattn_decode_selected; dims whose partial results need more than 16 MiB
 * ((320 + B * Hkv * T) x R x min(Tq * Hq / Hkv, 64) x (d + 2) x 4 bytes, T
 * = the 64-row tiles of a (request, KV head), R = 4 records per slot for
 * bf16 caches with Tq * Hq / Hkv <= 16, 2 for fp8 caches, 1 otherwise) are
 * rejected with SPATTN_ERR_UNSUPPORTED before anything is enqueued.  No
 * allocation call is made.  The first call on each device looks up the array's device address
 * (a host-side CUDA runtime call), so make that first call before any stream
 * capture.  Every call on a device shares the one array and leaves its
 * contents behind; calls whose executions overlap on the GPU (different
 * streams, or graphs replayed concurrently) race on it and give undefined
 * results, so serialise them.
 */
spattn_status spattn_decode_selected_noalloc(const spattn_dims *dims, const spattn_params *params,
                                             const void *q, const void *k_cache, const void *v_cache,
                                             const float *k_scale, const float *v_scale,
                                             const int32_t *block_table, const int32_t *seq_lens,
                                             const int32_t *sel_idx, const int32_t *sel_count,
                                             float *out, spattn_stream_t stream);

/*
 * spattn_decode -- the whole decode step after the cache append:
 * block scores, selection, sparse attention and the split merge.
 * kbar must be current (spattn_compress_keys after each append).
 * sel_idx / sel_count receive the selection; scores_out (optional, may be
 * NULL) receives the block scores, otherwise they live in the workspace.
 */
spattn_status spattn_decode(const spattn_dims *dims, const spattn_params *params,
                            const void *q, const void *k_cache, const void *v_cache,
                            const float *k_scale, const float *v_scale,
                            const int32_t *block_table, const int32_t *seq_lens,
                            const void *kbar, float *out, int32_t *sel_idx,
                            int32_t *sel_count, float *scores_out, void *workspace,
                            size_t workspace_bytes, spattn_stream_t stream);

/* ================================================================ HCA branch
 *
 * The weight-free compressed branch ("CSA + HCA 混合注意力机制" §5.1-5.2): every
 * SPATTN_HCA_BLOCKS consecutive blocks (m' = 128 tokens) of a request are
 * pooled into one key entry and one value entry, and every query attends
 * densely over its request's visible entries (no selection).  Readings of
 * the page: the page's learned pooling is replaced by the mean over the
 * entry's filled tokens; an entry is visible to query token t when all its
 * tokens are at or before position seq_lens[b] - Tq + t; no position tag
 * and no learned sink logit.  The branch's output joins the sparse branch's
 * (spattn_decode_selected_lse) through spattn_lse_merge, which is softmax
 * attention over the union of both key sets.
 *
 * khat / vhat are device fp32 [B][Hkv][G][d] with G = spattn_hca_entries():
 * the entries of one (request, KV head) are contiguous, so that the dense
 * attention streams them in large copies.
 */
#define SPATTN_HCA_BLOCKS 2

/* G = ceil(max_blocks_per_seq / SPATTN_HCA_BLOCKS): entries per request in
 * the khat / vhat buffers.  Returns -1 on invalid dims. */
int32_t spattn_hca_entries(const spattn_dims *dims);

/*
 * spattn_hca_pool -- mean K and V of each entry.
 *
 * khat[b][h][g][:] = mean over the tokens [128 g, min(L, 128 (g + 1))) of
 * request b of K (dequantised with k_scale for fp8; fp32 sums), vhat the same
 * of V.  With old_lens == NULL every entry of every request is written
 * (entries past the end of a request: zeros); otherwise only the entries
 * that hold a token of [old_lens[b], seq_lens[b]).  k_scale / v_scale may be
 * NULL for bf16 caches.  Block-table entries outside the pool are skipped
 * and set SPATTN_DEV_BAD_PAGE; a bad seq_len sets SPATTN_DEV_BAD_LEN.
 */
spattn_status spattn_hca_pool(const spattn_dims *dims, const void *k_cache, const void *v_cache,
                              const float *k_scale, const float *v_scale,
                              const int32_t *block_table, const int32_t *old_lens,
                              const int32_t *seq_lens, float *khat, float *vhat,
                              spattn_stream_t stream);

/* Bytes of workspace spattn_hca_attend / spattn_hca_attend_merge need (the
 * partial results of the shares of each request's entries).  Returns 0 on
 * invalid dims. */
size_t spattn_hca_workspace_size(const spattn_dims *dims);

/*
 * spattn_hca_attend -- dense attention over the pooled entries.
 *
 * out[b][t][i][:] = softmax_g(sm_scale * q . khat[b][h][g]) vhat[b][h][g]
 * over the visible entries g of (b, t), h = i / (Hq / Hkv); lse[b][t][i] =
 * ln of the softmax's denominator.  A row with no visible entry gets zeros
 * and -inf.  fp32 throughout; out and lse are device [B][Tq][Hq][d] and
 * [B][Tq][Hq] (both required).  workspace: device, 256-byte aligned, at
 * least spattn_hca_workspace_size() bytes (SPATTN_ERR_WORKSPACE otherwise);
 * its contents need no initialisation.
 */
spattn_status spattn_hca_attend(const spattn_dims *dims, const spattn_params *params,
                                const void *q, const float *khat, const float *vhat,
                                const int32_t *seq_lens, float *out, float *lse,
                                void *workspace, size_t workspace_bytes,
                                spattn_stream_t stream);

/*
 * spattn_hca_attend_merge -- spattn_hca_attend with the merge of
 * spattn_lse_merge folded into its last kernel: out / lse = the softmax over
 * the visible entries and another branch's keys together, given that
 * branch's out_other ([B][Tq][Hq][d]) and lse_other ([B][Tq][Hq], as
 * spattn_decode_selected_lse writes them).  lse may be NULL.  out and lse
 * may be out_other and lse_other.  Workspace as spattn_hca_attend.
 */
spattn_status spattn_hca_attend_merge(const spattn_dims *dims, const spattn_params *params,
                                      const void *q, const float *khat, const float *vhat,
                                      const int32_t *seq_lens, const float *out_other,
                                      const float *lse_other, float *out, float *lse,
                                      void *workspace, size_t workspace_bytes,
                                      spattn_stream_t stream);

/*
 * spattn_lse_merge -- one softmax over two disjoint key sets from the two
 * partial results (B * Tq * Hq rows of d):
 *   out = (e^lse_a out_a + e^lse_b out_b) / (e^lse_a + e^lse_b),
 *   lse = ln(e^lse_a + e^lse_b)   (lse may be NULL).
 * A row whose two lse are -inf gets zeros and -inf.  out / lse may be the
 * same buffers as out_a / lse_a or out_b / lse_b.  Device fp32 pointers.
 * Of dims only batch, q_tokens, num_q_heads and head_dim (128) are read.
 */
spattn_status spattn_lse_merge(const spattn_dims *dims, const float *out_a, const float *lse_a,
                               const float *out_b, const float *lse_b, float *out, float *lse,
                               spattn_stream_t stream);

/* Message for the last failed call on this host thread ("" if none). */
const char *spattn_last_error(void);

/* Synchronises `stream`, copies the current device's status word to
 * *host_out (host pointer) and clears it.  Returns SPATTN_OK when the copy
 * worked (whatever the word holds). */
spattn_status spattn_get_device_status(int32_t *host_out, spattn_stream_t stream);

/* Library version string, e.g. "spattn 0.1 sm_100a". */
const char *spattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPATTN_H */
