// select.cuh -- keep sink + local + the best middle blocks per (b, KV head).
//
// "Claude Opus 长上下文 KV Cache 稀疏注意力", §稀疏注意力与 KV Cache 压缩的工程实现:
// blocks are the unit of retention; the first block (attention sink) and the
// most recent blocks (local context) are always kept; middle blocks are kept
// by Top-P over their importance.  "CSA + HCA 混合注意力机制" §4.4 step 3:
// top-k of the scores.  Ranking: score descending, equal scores by lower
// block id.  Top-p: the shortest prefix of the ranking whose softmax mass
// (over the middle blocks) reaches p, cut to k_max = floor(ratio * n_mid).
//
// The top-k cut is found by bucketing the scores by value between the row's
// min and max (2048 buckets, monotone in the score), so that every block in a
// bucket above the crossing bucket is in, and ranking the few blocks of the
// crossing bucket exactly by (score, index).  Rows whose crossing bucket is
// crowded (many equal scores) fall back to a 3-pass radix select on the
// order-preserving uint32 keys.
#pragma once

#include "common.cuh"

namespace spattn {

struct SelectArgs {
    const float *scores;       // [B][Tq][Hkv][max_blocks]
    const int32_t *seq_lens;
    int32_t *sel_idx;          // [B][Hkv][max_sel]
    int32_t *sel_count;        // [B][Hkv]
    int tq, hkv, max_blocks, max_sel, sink, local, mode, top_k;
    float top_p, max_ratio, min_ratio;
    int n_mid_cap;             // keys capacity (>= every row's middle count)
    int sort_cap;              // power-of-two sort capacity (top-p), else 0
    int len_early;             // the kernel before this one is the scoring grid of the same decode call
};

constexpr int kSelThreads = 1024;
constexpr int kBuckets = 2048;
constexpr int kCand = 256;     // largest crossing bucket ranked exactly

struct SelectShared {
    unsigned long long *sortbuf;  // [sort_cap]
    uint32_t *keys;            // [n_mid_cap]
    uint32_t *hist;            // [kBuckets]
    uint32_t *cand_key;        // [kCand]
    int *cand_idx;             // [kCand]
    int *cand_ok;              // [kCand]
    int *itmp;                 // [72]
    float *ftmp;               // [40]
    int *misc;                 // [8]
    uint8_t *flags;            // [max_blocks]
};

__host__ __device__ inline size_t select_smem_bytes(int n_mid_cap, int sort_cap, int max_blocks) {
    size_t b = 0;
    b += (size_t)sort_cap * 8;
    b += (size_t)n_mid_cap * 4;
    b += kBuckets * 4 + 3 * kCand * 4 + 72 * 4 + 40 * 4 + 8 * 4;
    b += ((size_t)max_blocks + 15) / 16 * 16;
    return b;
}

// ------------------------------------------------------------ block helpers

// Block-wide max and min of one uint32 per thread (every thread calls it):
// per-warp reductions, then every warp reduces the warps' results.
__device__ __forceinline__ void block_minmax_u32(uint32_t vmax, uint32_t vmin, int *tmp, uint32_t &omax,
                                                 uint32_t &omin) {
    vmax = __reduce_max_sync(0xffffffffu, vmax);
    vmin = __reduce_min_sync(0xffffffffu, vmin);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) {
        tmp[threadIdx.x >> 5] = (int)vmax;
        tmp[32 + (threadIdx.x >> 5)] = (int)vmin;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    omax = __reduce_max_sync(0xffffffffu, lane < nw ? (uint32_t)tmp[lane] : 0u);
    omin = __reduce_min_sync(0xffffffffu, lane < nw ? (uint32_t)tmp[32 + lane] : 0xffffffffu);
}

// Block-wide sum of one float per thread: per-warp butterflies, then a
// butterfly over the warps' sums (the same fixed order on every run; every
// lane ends with the same bits).
__device__ __forceinline__ float block_sum_f(float v, float *tmp) {
    v = warp_sum(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) tmp[threadIdx.x >> 5] = v;
    __syncthreads();
    const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    return warp_sum(lane < nw ? tmp[lane] : 0.f);
}

// Middle scores of a row -> order-preserving keys in shared memory.  The
// row buffer has n_cap >= n readable columns, so the loads of a thread (16
// at a time) need not wait for n.  Returns the thread's max/min key over i < n.
__device__ __forceinline__ void load_keys(const SelectShared &sh, const float *row, int n_cap,
                                          const int *n_ptr, uint32_t &kmax, uint32_t &kmin) {
    kmax = 0;
    kmin = 0xffffffffu;
    for (int i0 = threadIdx.x; i0 < n_cap; i0 += 16 * blockDim.x) {
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = i0 + u * blockDim.x;
            v[u] = i < n_cap ? row[i] : 0.f;
        }
        const int n = *n_ptr;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < n) {
                const uint32_t key = float_key(v[u]);
                sh.keys[i] = key;
                kmax = max(kmax, key);
                kmin = min(kmin, key);
            }
        }
    }
}

// Histogram bins in descending order, 2048 / blockDim consecutive per
// thread: the bin holding the kk-th element from the top, the count of all
// elements in higher bins, and the bin's own count (misc[0..2]).
__device__ void find_crossing(const SelectShared &sh, int nbins, int kk) {
    const int bpt = kBuckets / blockDim.x;
    const int p0 = threadIdx.x * bpt;
    int mine = 0;
    for (int q = 0; q < bpt; ++q)
        if (p0 + q < nbins) mine += (int)sh.hist[nbins - 1 - p0 - q];
    int tot;
    int ex = block_excl_scan(mine, sh.itmp, &tot);
    if (ex < kk && kk <= ex + mine) {
        for (int q = 0; q < bpt; ++q) {
            const int c = (int)sh.hist[nbins - 1 - p0 - q];
            if (kk <= ex + c) {
                sh.misc[0] = nbins - 1 - p0 - q;
                sh.misc[1] = ex;
                sh.misc[2] = c;
                break;
            }
            ex += c;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- the cut

// The top k of a row (1 <= k < n): either "bucket" form -- every element in
// a bucket above `bstar`, plus the crossing bucket's candidates flagged in
// cand_ok -- or "radix" form -- every key above T plus the first need_eq keys
// equal to T by index.
struct Cut {
    bool bucket;
    float smin, inv;
    int bstar, ncand;
    uint32_t T;
    int need_eq, cnt_eq;
};

__device__ __forceinline__ int bucket_of(float s, float smin, float inv) {
    const int b = (int)((s - smin) * inv);  // monotone non-decreasing in s
    return min(max(b, 0), kBuckets - 1);
}

// k-th largest key by a 3-pass most-significant-digit radix select
// (11 + 11 + 10 bits): the key T, how many keys equal to T belong to the
// top k, and how many keys equal T in all.
__device__ void radix_select(const SelectShared &sh, int n, int k, uint32_t &T, int &need_eq, int &cnt_eq) {
    uint32_t prefix = 0, mask = 0;
    int kk = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nbins = pass < 2 ? 2048 : 1024;
        for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) sh.hist[i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += blockDim.x) {
            const int i = i0 + threadIdx.x;
            uint32_t digit = 0xffffffffu;
            if (i < n) {
                const uint32_t key = sh.keys[i];
                if ((key & mask) == prefix) digit = (key >> shift) & (nbins - 1);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (digit != 0xffffffffu && (threadIdx.x & 31) == __ffs(peers) - 1)
                atomicAdd(&sh.hist[digit], (uint32_t)__popc(peers));
        }
        __syncthreads();
        find_crossing(sh, nbins, kk);
        prefix |= (uint32_t)sh.misc[0] << shift;
        mask |= (uint32_t)(nbins - 1) << shift;
        kk -= sh.misc[1];
        cnt_eq = sh.misc[2];
        __syncthreads();
    }
    T = prefix;
    need_eq = kk;
}

// Visit the radix-form set {key > T} + {the first need_eq keys == T by
// index} (contiguous index range per thread, one block scan).
template <typename Fn>
__device__ void for_each_radix_chosen(const SelectShared &sh, int n, uint32_t T, int need_eq, Fn fn) {
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    int ceq = 0;
    for (int i = lo; i < hi; ++i) ceq += sh.keys[i] == T;
    int tot;
    int eq_before = block_excl_scan(ceq, sh.itmp, &tot);
    for (int i = lo; i < hi; ++i) {
        const uint32_t key = sh.keys[i];
        if (key > T || (key == T && eq_before++ < need_eq)) fn(i);
    }
}

// Every element of the cut, in no particular order, once: fn(i).
template <typename Fn>
__device__ void for_each_in_cut(const SelectShared &sh, int n, const Cut &cut, Fn fn) {
    if (cut.bucket) {
        for (int i = threadIdx.x; i < n; i += blockDim.x)
            if (bucket_of(key_float(sh.keys[i]), cut.smin, cut.inv) > cut.bstar) fn(i);
        for (int t = threadIdx.x; t < cut.ncand; t += blockDim.x)
            if (sh.cand_ok[t]) fn(sh.cand_idx[t]);
    } else if (cut.need_eq == cut.cnt_eq) {
        for (int i = threadIdx.x; i < n; i += blockDim.x)
            if (sh.keys[i] >= cut.T) fn(i);
    } else {
        for_each_radix_chosen(sh, n, cut.T, cut.need_eq, fn);
    }
}

// The cut of the top k, and on_cut(i) called once for every element of it
// (in no particular order).  on_each(i, key) is called once for every
// element, in the order i = tid, tid + blockDim, ..., if and only if the
// bucket form is tried; returns whether it was.  Bucket form: one histogram
// pass (with on_each), then one pass that hands the elements of the buckets
// above the crossing one to on_cut and gathers the crossing bucket, whose
// candidates are ranked exactly by (key desc, index asc) and handed over by
// thread t for candidate t.
template <typename EachFn, typename CutFn>
__device__ Cut find_cut(const SelectShared &sh, int n, int k, uint32_t kmax, uint32_t kmin, EachFn on_each,
                        CutFn on_cut, bool *each_called) {
    Cut cut{};
    *each_called = false;
    const float smax = key_float(kmax), smin = key_float(kmin);
    if (isfinite(smax) && isfinite(smin) && smax > smin) {
        *each_called = true;
        cut.smin = smin;
        cut.inv = (float)kBuckets / (smax - smin);
        for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) sh.hist[i] = 0;
        if (threadIdx.x == 0) sh.misc[3] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = sh.keys[i];
            on_each(i, key);
            atomicAdd(&sh.hist[bucket_of(key_float(key), cut.smin, cut.inv)], 1u);
        }
        __syncthreads();
        find_crossing(sh, kBuckets, k);
        cut.bstar = sh.misc[0];
        const int need = k - sh.misc[1], c = sh.misc[2];
        if (c <= kCand) {
            cut.bucket = true;
            cut.ncand = c;
            // the buckets above the crossing one go to on_cut; the crossing
            // bucket is gathered
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const uint32_t key = sh.keys[i];
                const int bk = bucket_of(key_float(key), cut.smin, cut.inv);
                if (bk > cut.bstar) {
                    on_cut(i);
                } else if (bk == cut.bstar) {
                    const int slot = atomicAdd(&sh.misc[3], 1);
                    sh.cand_key[slot] = key;
                    sh.cand_idx[slot] = i;
                }
            }
            __syncthreads();
            // rank candidate t by four lanes of a warp, each over a quarter
            // of the candidates (the warp's lanes stay together)
            for (int base = threadIdx.x & ~31; base < 4 * c; base += blockDim.x) {
                const int t4 = base + (threadIdx.x & 31);
                const int t = t4 >> 2, part = t4 & 3;
                int rank = 0;
                if (t < c) {
                    const uint32_t kt = sh.cand_key[t];
                    const int it = sh.cand_idx[t];
                    const int u_lo = part * c / 4, u_hi = (part + 1) * c / 4;
#pragma unroll 4
                    for (int u = u_lo; u < u_hi; ++u) {
                        const uint32_t ku = sh.cand_key[u];
                        rank += ku > kt || (ku == kt && sh.cand_idx[u] < it);
                    }
                }
                rank += __shfl_xor_sync(0xffffffffu, rank, 1);
                rank += __shfl_xor_sync(0xffffffffu, rank, 2);
                if (t < c && part == 0) sh.cand_ok[t] = rank < need;
            }
            __syncthreads();
            for (int t = threadIdx.x; t < c; t += blockDim.x)
                if (sh.cand_ok[t]) on_cut(sh.cand_idx[t]);
            return cut;
        }
    }
    cut.bucket = false;
    radix_select(sh, n, k, cut.T, cut.need_eq, cut.cnt_eq);
    for_each_in_cut(sh, n, cut, on_cut);
    return cut;
}

__device__ void bitonic_sort_desc(unsigned long long *buf, int N) {
    for (int size = 2; size <= N; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (N >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long x = buf[lo], y = buf[hi];
                if ((x < y) == desc) {
                    buf[lo] = y;
                    buf[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

// Carve the dynamic shared memory of a selection CTA.
__device__ __forceinline__ SelectShared select_shared(const SelectArgs &a, unsigned long long *base) {
    SelectShared sh;
    char *p = reinterpret_cast<char *>(base);
    sh.sortbuf = reinterpret_cast<unsigned long long *>(p);
    p += (size_t)a.sort_cap * 8;
    sh.keys = reinterpret_cast<uint32_t *>(p);
    p += (size_t)a.n_mid_cap * 4;
    sh.hist = reinterpret_cast<uint32_t *>(p);
    p += kBuckets * 4;
    sh.cand_key = reinterpret_cast<uint32_t *>(p);
    p += kCand * 4;
    sh.cand_idx = reinterpret_cast<int *>(p);
    p += kCand * 4;
    sh.cand_ok = reinterpret_cast<int *>(p);
    p += kCand * 4;
    sh.itmp = reinterpret_cast<int *>(p);
    p += 72 * 4;
    sh.ftmp = reinterpret_cast<float *>(p);
    p += 40 * 4;
    sh.misc = reinterpret_cast<int *>(p);
    p += 8 * 4;
    sh.flags = reinterpret_cast<uint8_t *>(p);
    return sh;
}

// A row's length, checked (a bad one counts as empty and is reported).
__device__ __forceinline__ int checked_len(const SelectArgs &a, int L) {
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0) flag(SPATTN_DEV_BAD_LEN);
        return 0;
    }
    return L;
}

// k_max = floor(ratio * n_mid), the product taken in double so that an
// integral product is not rounded below the integer.
__device__ __forceinline__ int select_k_max(const SelectArgs &a, int n_mid) {
    return a.max_ratio > 0.f ? min(n_mid, (int)floor((double)a.max_ratio * (double)n_mid)) : n_mid;
}

// The kept middle blocks of query token t of row (b, h): sh.flags[S + i] = 1
// for each (other flags untouched).  Every thread of the CTA calls it; it
// ends with a barrier.
__device__ void select_token(const SelectShared &sh, const SelectArgs &a, int b, int h, int t, int nb, int n_mid) {
    const int S = a.sink, W = a.local;
    const int k_max = select_k_max(a, n_mid);
    const int k_topk = a.top_k > 0 ? min(a.top_k, k_max) : k_max;
    const float *row = a.scores + (((int64_t)b * a.tq + t) * a.hkv + h) * a.max_blocks + S;
    const bool anchor = a.mode == SPATTN_SEL_TOPP_ANCHOR;
    int k = a.mode == SPATTN_SEL_TOPK ? k_topk : k_max;
    if (k <= 0 && !anchor) return;
    if (a.mode == SPATTN_SEL_TOPK && k >= n_mid) {
        for (int i = threadIdx.x; i < n_mid; i += blockDim.x) sh.flags[S + i] = 1;
        __syncthreads();
        return;
    }
    uint32_t kmax_l, kmin_l, kmax, kmin;
    load_keys(sh, row, a.n_mid_cap, &n_mid, kmax_l, kmin_l);
    block_minmax_u32(kmax_l, kmin_l, sh.itmp, kmax, kmin);
    if (anchor) {
        // cap from the anchors: a = their best score, hi / lo the middle's
        // extremes; r = clamp((hi - a) / (hi - lo), 0, 1), ratio = min_ratio
        // + r * (max_ratio - min_ratio), k = floor(ratio * n_mid), all in
        // double with separately rounded operations
        const float *full = row - S;
        float amax = -INFINITY;
        for (int j = 0; j < S; ++j) amax = fmaxf(amax, full[j]);       // n_mid > 0: nb > S + W
        for (int j = nb - W; j < nb; ++j) amax = fmaxf(amax, full[j]);
        const double hi = (double)key_float(kmax), lo = (double)key_float(kmin);
        double r = hi > lo ? __ddiv_rn(__dsub_rn(hi, (double)amax), __dsub_rn(hi, lo)) : 0.0;
        r = r < 0.0 ? 0.0 : (r > 1.0 ? 1.0 : r);
        const double ratio =
            __dadd_rn((double)a.min_ratio, __dmul_rn(r, __dsub_rn((double)a.max_ratio, (double)a.min_ratio)));
        k = min(n_mid, (int)floor(__dmul_rn(ratio, (double)n_mid)));
        if (k <= 0) {
            __syncthreads();
            return;
        }
    }
    bool each_called;
    if (a.mode == SPATTN_SEL_TOPK) {
        find_cut(sh, n_mid, k, kmax, kmin, [](int, uint32_t) {}, [&](int i) { sh.flags[S + i] = 1; },
                 &each_called);
        __syncthreads();
        return;
    }
    // top-p: probabilities are the softmax of the middle scores; the
    // normaliser's terms are summed in the histogram pass when there is one
    const float smax = key_float(kmax);
    float z = 0.f, mk = 0.f;
    Cut cut{};
    each_called = false;
    if (k < n_mid)   // mass of the k_max best blocks (mk) with the cut
        cut = find_cut(
            sh, n_mid, k, kmax, kmin, [&](int, uint32_t key) { z += expf(key_float(key) - smax); },
            [&](int i) { mk += expf(key_float(sh.keys[i]) - smax); }, &each_called);
    if (!each_called)
        for (int i = threadIdx.x; i < n_mid; i += blockDim.x) z += expf(key_float(sh.keys[i]) - smax);
    const float Z = block_sum_f(z, sh.ftmp);
    if (k < n_mid) {
        // below p, the cap decides alone
        const float mass = block_sum_f(mk, sh.ftmp) / Z;
        if (mass < a.top_p) {
            for_each_in_cut(sh, n_mid, cut, [&](int i) { sh.flags[S + i] = 1; });
            __syncthreads();
            return;
        }
    }
    // the shortest prefix reaching p lies within the k candidates: sort them
    int npow = 1;
    while (npow < k) npow <<= 1;
    for (int i = threadIdx.x; i < npow; i += blockDim.x) sh.sortbuf[i] = 0ull;
    if (threadIdx.x == 0) sh.misc[4] = 0;
    __syncthreads();
    auto put = [&](int i) {
        const int slot = atomicAdd(&sh.misc[4], 1);
        sh.sortbuf[slot] = ((unsigned long long)sh.keys[i] << 32) | (0xffffffffu - (uint32_t)(S + i));
    };
    if (k < n_mid)
        for_each_in_cut(sh, n_mid, cut, put);
    else
        for (int i = threadIdx.x; i < n_mid; i += blockDim.x) put(i);
    __syncthreads();
    bitonic_sort_desc(sh.sortbuf, npow);
    if (threadIdx.x == 0) sh.misc[5] = k;  // first crossing (default: all k)
    __syncthreads();
    const int per = (k + blockDim.x - 1) / blockDim.x;
    const int lo = min(k, (int)threadIdx.x * per), hi = min(k, lo + per);
    float local = 0.f;
    for (int i = lo; i < hi; ++i) local += expf(key_float((uint32_t)(sh.sortbuf[i] >> 32)) - smax) / Z;
    float c = block_incl_scan_f(local, sh.ftmp) - local;
    for (int i = lo; i < hi; ++i) {
        c += expf(key_float((uint32_t)(sh.sortbuf[i] >> 32)) - smax) / Z;
        if (c >= a.top_p) {
            atomicMin(&sh.misc[5], i + 1);
            break;
        }
    }
    __syncthreads();
    const int m = sh.misc[5];
    for (int i = threadIdx.x; i < m; i += blockDim.x)
        sh.flags[0xffffffffu - (uint32_t)(sh.sortbuf[i] & 0xffffffffull)] = 1;
    __syncthreads();
}

// Kept flags sh.flags[0, nb) -> ascending block ids of row bh.  Warp w
// takes a run of consecutive 32-flag chunks (lane = flag, counted by
// ballots); one scan over the warps' counts places the runs.
__device__ void compact_flags(const SelectShared &sh, const SelectArgs &a, int bh, int nb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nchunks = (nb + 31) >> 5;
    const int per = (nchunks + nw - 1) / nw;
    const int ch_lo = min(nchunks, warp * per), ch_hi = min(nchunks, ch_lo + per);
    int cnt = 0;
    for (int ch = ch_lo; ch < ch_hi; ++ch) {
        const int j = ch * 32 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, j < nb && sh.flags[j]));
    }
    // (itmp is free: the caller's last barrier ended its previous use)
    if (lane == 0) sh.itmp[warp] = cnt;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < nw ? sh.itmp[lane] : 0;
        const int inc = warp_incl_scan(v);
        __syncwarp();
        if (lane < nw) sh.itmp[lane] = inc - v;
        if (lane == 31) sh.itmp[32] = inc;
    }
    __syncthreads();
    int pos = sh.itmp[warp];
    const int total = sh.itmp[32];
    int32_t *dst = a.sel_idx + (int64_t)bh * a.max_sel;
    const unsigned below = (1u << lane) - 1u;
    for (int ch = ch_lo; ch < ch_hi; ++ch) {
        const int j = ch * 32 + lane;
        const bool f = j < nb && sh.flags[j];
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const int p = pos + __popc(bal & below);
        if (f && p < a.max_sel) dst[p] = j;
        pos += __popc(bal);
    }
    if (threadIdx.x == 0) {
        if (total > a.max_sel) flag(SPATTN_DEV_SEL_OVERFLOW);
        a.sel_count[bh] = min(total, a.max_sel);
    }
}

// Grid (B * Hkv), block 256 / 512 / 1024 threads (longer rows, more): one
// row, its query tokens one after another, the union compacted.
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    extern __shared__ unsigned long long smem_u64[];
    const SelectShared sh = select_shared(a, smem_u64);
    const int bh = blockIdx.x;
    const int b = bh / a.hkv, h = bh % a.hkv;
    // Launched early (programmatic dependent launch): nothing the kernel
    // before it may write is read before the wait.  Behind the scoring grid
    // of the same decode call (len_early), which does not write the lengths
    // and itself started after every earlier kernel had finished, the
    // length is loaded before the wait.
    int L = a.len_early ? a.seq_lens[b] : 0;
    // the lines (and translations) the kernel reads and writes, before the wait
    if (threadIdx.x < 32) {
        const int64_t last = (int64_t)a.tq * a.hkv * a.max_blocks - a.hkv * a.max_blocks;   // last token's row
        const void *p[6] = {a.sel_idx + (int64_t)bh * a.max_sel, a.sel_idx + (int64_t)bh * a.max_sel + a.max_sel - 1,
                            a.sel_count + bh, a.seq_lens + b,
                            a.scores + ((int64_t)b * a.tq * a.hkv + h) * a.max_blocks,
                            a.scores + ((int64_t)b * a.tq * a.hkv + h) * a.max_blocks + last + a.max_blocks - 1};
        if (threadIdx.x < 6 && a.max_sel > 0) prefetch_l2(p[threadIdx.x]);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!a.len_early) L = a.seq_lens[b];
    // the first token's score row into L1
    {
        const float *row0 = a.scores + ((int64_t)b * a.tq * a.hkv + h) * a.max_blocks;
        for (int i = threadIdx.x * 32; i < a.n_mid_cap + a.sink; i += blockDim.x * 32)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(row0 + i));
    }
    L = checked_len(a, L);
    const int nb = (L + kBlock - 1) / kBlock;
    const int S = a.sink, W = a.local;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) sh.flags[j] = (j < S || j >= nb - W) ? 1 : 0;
    const int n_mid = max(0, nb - S - W);
    __syncthreads();
    for (int t = 0; t < a.tq && n_mid > 0; ++t) select_token(sh, a, b, h, t, nb, n_mid);
    __syncthreads();
    compact_flags(sh, a, bh, nb);
}

}  // namespace spattn
