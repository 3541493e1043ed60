// select.cuh -- keep sink + local + the best middle blocks per (b, KV head).
//
// "Claude Opus 长上下文 KV Cache 稀疏注意力", §稀疏注意力与 KV Cache 压缩的工程实现:
// blocks are the unit of retention; the first block (attention sink) and the
// most recent blocks (local context) are always kept; middle blocks are kept
// by Top-P over their importance.  "CSA + HCA 混合注意力机制" §4.4 step 3:
// top-k of the scores.  Ranking: score descending, equal scores by lower
// block id.  Top-p: the shortest prefix of the ranking whose softmax mass
// (over the middle blocks) reaches p, cut to k_max = floor(ratio * n_mid).
#pragma once

#include "common.cuh"

namespace spattn {

struct SelectArgs {
    const float *scores;       // [B][Tq][Hkv][max_blocks]
    const int32_t *seq_lens;
    int32_t *sel_idx;          // [B][Hkv][max_sel]
    int32_t *sel_count;        // [B][Hkv]
    int tq, hkv, max_blocks, max_sel, sink, local, mode, top_k;
    float top_p, max_ratio;
    int n_mid_cap;             // keys capacity (>= every row's middle count)
    int sort_cap;              // power-of-two sort capacity (top-p), else 0
};

constexpr int kSelThreads = 1024;

struct SelectShared {
    uint32_t *keys;            // [n_mid_cap]
    unsigned long long *sortbuf;  // [sort_cap]
    uint32_t *hist;            // [2048]
    int *itmp;                 // [40]
    float *ftmp;               // [40]
    int *misc;                 // [8]
    uint8_t *flags;            // [max_blocks]
};

__host__ __device__ inline size_t select_smem_bytes(int n_mid_cap, int sort_cap, int max_blocks) {
    size_t b = 0;
    b += (size_t)sort_cap * 8;
    b += (size_t)n_mid_cap * 4;
    b += 2048 * 4 + 40 * 4 + 40 * 4 + 8 * 4;
    b += ((size_t)max_blocks + 15) / 16 * 16;
    return b;
}

// k-th largest key (1 <= k <= n) by a 3-pass most-significant-digit radix
// select (11 + 11 + 10 bits).  Returns the key T and how many elements equal
// to T belong to the top k (the rest of the top k is strictly greater).
__device__ void radix_select(const SelectShared &sh, int n, int k, uint32_t &T, int &need_eq) {
    uint32_t prefix = 0, mask = 0;
    int kk = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nbins = pass < 2 ? 2048 : 1024;
        for (int i = threadIdx.x; i < 2048; i += blockDim.x) sh.hist[i] = 0;
        __syncthreads();
        // scores crowd into few digits: lanes with equal digits add once
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
        // bins in descending digit order, two per thread
        const int i0 = 2 * threadIdx.x;
        const int c0 = i0 < nbins ? (int)sh.hist[nbins - 1 - i0] : 0;
        const int c1 = i0 + 1 < nbins ? (int)sh.hist[nbins - 2 - i0] : 0;
        int tot;
        const int ex = block_excl_scan(c0 + c1, sh.itmp, &tot);
        if (ex < kk && kk <= ex + c0) {
            sh.misc[0] = nbins - 1 - i0;
            sh.misc[1] = ex;
        } else if (ex + c0 < kk && kk <= ex + c0 + c1) {
            sh.misc[0] = nbins - 2 - i0;
            sh.misc[1] = ex + c0;
        }
        __syncthreads();
        prefix |= (uint32_t)sh.misc[0] << shift;
        mask |= (uint32_t)(nbins - 1) << shift;
        kk -= sh.misc[1];
        __syncthreads();
    }
    T = prefix;
    need_eq = kk;
}

// Visit the top-k set {key > T} + {the first need_eq keys == T by index} in
// index order.  Each thread owns a contiguous index range; fn(i, slot) gets
// the element's rank among the chosen elements in index order.
template <typename Fn>
__device__ void for_each_chosen(const SelectShared &sh, int n, uint32_t T, int need_eq, Fn fn) {
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    int ceq = 0, csel = 0;
    for (int i = lo; i < hi; ++i) {
        const uint32_t key = sh.keys[i];
        ceq += key == T;
    }
    int tot;
    int eq_before = block_excl_scan(ceq, sh.itmp, &tot);
    {
        int e = eq_before;
        for (int i = lo; i < hi; ++i) {
            const uint32_t key = sh.keys[i];
            if (key > T || (key == T && e++ < need_eq)) ++csel;
        }
    }
    int sel_before = block_excl_scan(csel, sh.itmp, &tot);
    for (int i = lo; i < hi; ++i) {
        const uint32_t key = sh.keys[i];
        if (key > T || (key == T && eq_before++ < need_eq)) fn(i, sel_before++);
    }
}

// Block-wide max of one uint32 per thread (every thread calls it).
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, int *tmp) {
    v = __reduce_max_sync(0xffffffffu, v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) tmp[threadIdx.x >> 5] = (int)v;
    __syncthreads();
    uint32_t r = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, (uint32_t)tmp[w]);
    return r;
}

// Block-wide sum of one float per thread, added in a fixed order.
__device__ __forceinline__ float block_sum_f(float v, float *tmp) {
    v = warp_sum(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) tmp[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += tmp[w];
    return r;
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

// Grid (B * Hkv), block kSelThreads.
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
    extern __shared__ unsigned long long smem_u64[];
    SelectShared sh;
    {
        char *p = reinterpret_cast<char *>(smem_u64);
        sh.sortbuf = reinterpret_cast<unsigned long long *>(p);
        p += (size_t)a.sort_cap * 8;
        sh.keys = reinterpret_cast<uint32_t *>(p);
        p += (size_t)a.n_mid_cap * 4;
        sh.hist = reinterpret_cast<uint32_t *>(p);
        p += 2048 * 4;
        sh.itmp = reinterpret_cast<int *>(p);
        p += 40 * 4;
        sh.ftmp = reinterpret_cast<float *>(p);
        p += 40 * 4;
        sh.misc = reinterpret_cast<int *>(p);
        p += 8 * 4;
        sh.flags = reinterpret_cast<uint8_t *>(p);
    }
    const int bh = blockIdx.x;
    const int b = bh / a.hkv, h = bh % a.hkv;
    int L = a.seq_lens[b];
    if (L < 0 || L > a.max_blocks * kBlock) {
        if (threadIdx.x == 0) flag(SPATTN_DEV_BAD_LEN);
        L = 0;
    }
    const int nb = (L + kBlock - 1) / kBlock;
    const int S = a.sink, W = a.local;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) sh.flags[j] = (j < S || j >= nb - W) ? 1 : 0;
    const int n_mid = max(0, nb - S - W);
    // k_max = floor(ratio * n_mid), the product taken in double so that an
    // integral product is not rounded below the integer.
    const int k_max =
        a.max_ratio > 0.f ? min(n_mid, (int)floor((double)a.max_ratio * (double)n_mid)) : n_mid;
    const int k_topk = a.top_k > 0 ? min(a.top_k, k_max) : k_max;
    __syncthreads();

    for (int t = 0; t < a.tq && n_mid > 0; ++t) {
        const float *row = a.scores + (((int64_t)b * a.tq + t) * a.hkv + h) * a.max_blocks + S;
        if (a.mode == SPATTN_SEL_TOPK) {
            if (k_topk >= n_mid) {
                for (int i = threadIdx.x; i < n_mid; i += blockDim.x) sh.flags[S + i] = 1;
                __syncthreads();
                continue;
            }
            if (k_topk <= 0) continue;
            for (int i = threadIdx.x; i < n_mid; i += blockDim.x) sh.keys[i] = float_key(row[i]);
            __syncthreads();
            uint32_t T;
            int need_eq;
            radix_select(sh, n_mid, k_topk, T, need_eq);
            for_each_chosen(sh, n_mid, T, need_eq, [&](int i, int) { sh.flags[S + i] = 1; });
            __syncthreads();
            continue;
        }
        // top-p: probabilities are the softmax of the middle scores
        if (k_max <= 0) continue;
        uint32_t kmax_local = 0;
        for (int i = threadIdx.x; i < n_mid; i += blockDim.x) {
            const uint32_t key = float_key(row[i]);
            sh.keys[i] = key;
            kmax_local = max(kmax_local, key);
        }
        const float smax = key_float(block_max_u32(kmax_local, sh.itmp));
        float z = 0.f;
        for (int i = threadIdx.x; i < n_mid; i += blockDim.x) z += expf(key_float(sh.keys[i]) - smax);
        const float Z = block_sum_f(z, sh.ftmp);
        const int kc = k_max;
        uint32_t T = 0;
        int need_eq = 0;
        if (kc < n_mid) {
            radix_select(sh, n_mid, kc, T, need_eq);
            // mass of the k_max best blocks: below p, the cap decides alone
            float mass = 0.f;
            for_each_chosen(sh, n_mid, T, need_eq,
                            [&](int i, int) { mass += expf(key_float(sh.keys[i]) - smax) / Z; });
            mass = block_sum_f(mass, sh.ftmp);
            if (mass < a.top_p) {
                for_each_chosen(sh, n_mid, T, need_eq, [&](int i, int) { sh.flags[S + i] = 1; });
                __syncthreads();
                continue;
            }
        }
        // the shortest prefix reaching p lies within the candidates: sort them
        int npow = 1;
        while (npow < kc) npow <<= 1;
        for (int i = threadIdx.x; i < npow; i += blockDim.x) sh.sortbuf[i] = 0ull;
        __syncthreads();
        auto put = [&](int i, int slot) {
            const uint32_t j = (uint32_t)(S + i);
            sh.sortbuf[slot] = ((unsigned long long)sh.keys[i] << 32) | (0xffffffffu - j);
        };
        if (kc < n_mid)
            for_each_chosen(sh, n_mid, T, need_eq, put);
        else
            for (int i = threadIdx.x; i < n_mid; i += blockDim.x) put(i, i);
        __syncthreads();
        bitonic_sort_desc(sh.sortbuf, npow);
        if (threadIdx.x == 0) sh.misc[2] = kc;  // first crossing (default: all kc)
        __syncthreads();
        const int per = (kc + blockDim.x - 1) / blockDim.x;
        const int lo = min(kc, (int)threadIdx.x * per), hi = min(kc, lo + per);
        float local = 0.f;
        for (int i = lo; i < hi; ++i) local += expf(key_float((uint32_t)(sh.sortbuf[i] >> 32)) - smax) / Z;
        float c = block_incl_scan_f(local, sh.ftmp) - local;
        for (int i = lo; i < hi; ++i) {
            c += expf(key_float((uint32_t)(sh.sortbuf[i] >> 32)) - smax) / Z;
            if (c >= a.top_p) {
                atomicMin(&sh.misc[2], i + 1);
                break;
            }
        }
        __syncthreads();
        const int m = sh.misc[2];
        for (int i = threadIdx.x; i < m; i += blockDim.x)
            sh.flags[0xffffffffu - (uint32_t)(sh.sortbuf[i] & 0xffffffffull)] = 1;
        __syncthreads();
    }
    __syncthreads();

    // compaction: ascending block ids
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int lo = min(nb, (int)threadIdx.x * per), hi = min(nb, lo + per);
    int cnt = 0;
    for (int j = lo; j < hi; ++j) cnt += sh.flags[j];
    int total;
    int pos = block_excl_scan(cnt, sh.itmp, &total);
    int32_t *dst = a.sel_idx + (int64_t)bh * a.max_sel;
    for (int j = lo; j < hi; ++j)
        if (sh.flags[j]) {
            if (pos < a.max_sel) dst[pos] = j;
            ++pos;
        }
    if (threadIdx.x == 0) {
        if (total > a.max_sel) flag(SPATTN_DEV_SEL_OVERFLOW);
        a.sel_count[bh] = min(total, a.max_sel);
    }
}

}  // namespace spattn
