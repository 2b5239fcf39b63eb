// tt_select.cuh - block-wide selection over 64-bit candidate keys, shared
// by the select kernels (K4) and the exact fallback scan.
//
// One CTA of K4_THREADS threads works on one list of distinct keys. The r-th
// largest key is found by a most-significant-digit radix select (digits of
// 11/11/10/11/11/10 bits, a 2048-bin shared-memory histogram per digit)
// until at most K4_THREADS keys share the selected prefix; those are ranked
// directly. The cost depends only on the number of keys, not on their order.
// (Order of results: score descending, ties by ascending id - mhtirogla.ai
// Two-tower retrieval, Code, Towers::top_k.)
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"

namespace tt {

constexpr int K4_THREADS = 256;
constexpr int K4_SORT_MAX = 2048;  // >= TT_MAX_K
constexpr int K4_BINS = 2048;
constexpr int K4_SMEM_KEYS = 4096;  // kept keys copied to shared memory when they fit

struct K4Smem {
    uint32_t hist[K4_BINS];
    uint32_t part[K4_THREADS];
    uint32_t above[K4_THREADS];
    uint64_t sorted[K4_SORT_MAX];
    uint64_t found_prefix;
    uint32_t found_remaining;
    uint32_t found_count;
    uint32_t n_collected;
    uint64_t result;
    uint64_t keys[K4_SMEM_KEYS];
};

// The query's kept keys: copied to shared memory when they fit, else read in place.
__device__ __forceinline__ const uint64_t* stage_keys(const uint64_t* __restrict__ g, int n, K4Smem& sm) {
    if (n > K4_SMEM_KEYS) return g;
    for (int i = threadIdx.x; i < n; i += K4_THREADS) sm.keys[i] = g[i];
    __syncthreads();
    return sm.keys;
}

// r-th largest (1-based, counting repeats) of n keys; 1 <= r <= n. Block-wide.
// Radix passes narrow the candidates to a digit prefix; once at most
// K4_THREADS keys share the prefix they are gathered and ranked directly.
__device__ inline uint64_t block_kth_largest(const uint64_t* keys, int n, int r, K4Smem& sm) {
    const int tid = threadIdx.x;
    // digits, most significant first: widths 11, 11, 10, 11, 11, 10
    uint64_t prefix = 0, mask = 0;
    uint32_t remaining = (uint32_t)r;
    int shift = 64;
#pragma unroll 1
    for (int pass = 0; pass < 6; ++pass) {
        const int w = (pass == 2 || pass == 5) ? 10 : 11;
        shift -= w;
        const int nb = 1 << w;
        for (int i = tid; i < nb; i += K4_THREADS) sm.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += K4_THREADS) {
            const uint64_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & (uint64_t)(nb - 1)], 1u);
        }
        __syncthreads();
        // Thread t owns bins [t*per, (t+1)*per); above[t] = count in higher bins.
        const int per = nb / K4_THREADS;
        uint32_t local = 0;
        for (int i = 0; i < per; ++i) local += sm.hist[tid * per + i];
        sm.part[tid] = local;
        __syncthreads();
        if (tid < 32) {
            uint32_t s = 0;
            for (int i = 0; i < 8; ++i) s += sm.part[tid * 8 + i];
            // suffix sum over lanes: sum of lanes > tid
            uint32_t incl = s;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, off);
                if (tid + off < 32) incl += v;
            }
            uint32_t run = incl - s;  // lanes above this one
            for (int i = 7; i >= 0; --i) {
                sm.above[tid * 8 + i] = run;
                run += sm.part[tid * 8 + i];
            }
        }
        __syncthreads();
        const uint32_t above = sm.above[tid];
        if (above < remaining && remaining <= above + local) {
            uint32_t run = above;
            for (int i = per - 1; i >= 0; --i) {
                const uint32_t c = sm.hist[tid * per + i];
                if (remaining <= run + c) {
                    sm.found_prefix = (uint64_t)(tid * per + i);
                    sm.found_remaining = remaining - run;
                    sm.found_count = c;
                    break;
                }
                run += c;
            }
        }
        __syncthreads();
        prefix |= sm.found_prefix << shift;
        mask |= (uint64_t)(nb - 1) << shift;
        remaining = sm.found_remaining;
        const uint32_t count = sm.found_count;
        __syncthreads();
        if (count <= (uint32_t)K4_THREADS) {
            // gather the keys with this prefix and rank them by counting
            if (tid == 0) sm.n_collected = 0;
            __syncthreads();
            for (int i = tid; i < n; i += K4_THREADS) {
                const uint64_t key = keys[i];
                if ((key & mask) == prefix) sm.sorted[atomicAdd(&sm.n_collected, 1u)] = key;
            }
            __syncthreads();
            if (tid < (int)count) {
                const uint64_t mine = sm.sorted[tid];
                uint32_t above_me = 0, equal = 0;
                for (uint32_t j = 0; j < count; ++j) {
                    above_me += sm.sorted[j] > mine;
                    equal += sm.sorted[j] == mine;
                }
                if (above_me < remaining && remaining <= above_me + equal) sm.result = mine;
            }
            __syncthreads();
            return sm.result;
        }
    }
    return prefix;
}

// The min(n_valid, k) largest of n keys, sorted descending, written as
// (id, score); slots past n_valid get (-1, -inf). The keys are distinct
// except for KEY_MIN entries (empty slots), and n_valid of them are not
// KEY_MIN. Block-wide; out_* point at one list's row of k entries.
__device__ inline void write_sorted_topk(const uint64_t* keys, int n, int n_valid, int k, K4Smem& sm,
                                         int32_t* out_ids, float* out_scores) {
    const int tid = threadIdx.x;
    const int r = n_valid < k ? n_valid : k;
    if (r > 0) {
        const uint64_t kth = block_kth_largest(keys, n, r, sm);
        if (tid == 0) sm.n_collected = 0;
        __syncthreads();
        // fewer than r keys are above the r-th largest; the rest of the r
        // slots hold it (one copy when keys are distinct)
        for (int i = tid; i < n; i += K4_THREADS) {
            const uint64_t key = keys[i];
            if (key > kth) {
                const uint32_t slot = atomicAdd(&sm.n_collected, 1u);
                if (slot < (uint32_t)r) sm.sorted[slot] = key;
            }
        }
        __syncthreads();
        const int above = (int)sm.n_collected < r ? (int)sm.n_collected : r;
        for (int i = above + tid; i < r; i += K4_THREADS) sm.sorted[i] = kth;
        __syncthreads();
        int P = 1;
        while (P < r) P <<= 1;
        for (int i = r + tid; i < P; i += K4_THREADS) sm.sorted[i] = KEY_MIN;
        __syncthreads();
        // bitonic sort, descending
        for (int size = 2; size <= P; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int i = tid; i < P; i += K4_THREADS) {
                    const int j = i ^ stride;
                    if (j > i) {
                        const uint64_t x = sm.sorted[i], y = sm.sorted[j];
                        const bool desc = (i & size) == 0;
                        if (desc ? (x < y) : (x > y)) {
                            sm.sorted[i] = y;
                            sm.sorted[j] = x;
                        }
                    }
                }
                __syncthreads();
            }
        }
    }
    for (int i = tid; i < k; i += K4_THREADS) {
        int32_t id = -1;
        float sc = -INFINITY;
        if (i < r) {
            id = (int32_t)key_id(sm.sorted[i]);
            sc = key_score(sm.sorted[i]);
        }
        out_ids[i] = id;
        out_scores[i] = sc;
    }
}

}  // namespace tt
