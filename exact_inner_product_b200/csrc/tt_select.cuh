// tt_select.cuh - block-wide selection over 64-bit candidate keys, shared
// by the select kernels (K4) and the exact fallback scan.
//
// One CTA of K4_THREADS threads works on one list of distinct keys. Up to
// 4096 keys and r <= 1024: a bucket select over linear score bins (below);
// where that cannot decide, for r <= K4_TOP_MAX, the best r keys kept sorted
// in registers (bitonic networks, below). Otherwise the r-th
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

// ---------------------------------------------------------------------------
// Top-r in registers (r <= K4_TOP_MAX). A warp holds 32 * KPL keys, element
// e = lane * KPL + j in register j of its lane. Bitonic networks (Batcher's
// sorting network) sort such a list with compare-exchanges inside a lane's
// registers (partner distance below KPL) or across lanes through shuffles.
// Two lists A and B sorted descending give the best 32 * KPL keys of their
// union as max(A[e], B[N - 1 - e]), a bitonic sequence that one cleaning
// cascade sorts. Every warp folds its chunks of the input into its own list
// this way; the warps' lists are then folded pairwise through shared memory.
// No shared-memory atomics and log2(8) block barriers, whatever the keys.
// ---------------------------------------------------------------------------
constexpr int K4_TOP_MAX = 256;

// One compare-exchange step of a bitonic network over the warp's list:
// elements e and e ^ D (D < KPL: both in this lane's registers), the larger
// first where (e & size) == 0.
template <int KPL, int D>
__device__ __forceinline__ void bitonic_in_lane(uint64_t (&v)[KPL], int size) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        if (j & D) continue;
        const bool desc = ((lane * KPL + j) & size) == 0;
        const uint64_t x = v[j], y = v[j | D];
        const bool swap = desc ? x < y : x > y;
        v[j] = swap ? y : x;
        v[j | D] = swap ? x : y;
    }
}

// The same step for d >= KPL: the partner element sits in register j of lane
// lane ^ (d / KPL).
template <int KPL>
__device__ __forceinline__ void bitonic_across(uint64_t (&v)[KPL], int size, int d) {
    const int lane = threadIdx.x & 31;
    const int ld = d / KPL;
    const bool lower = (lane & ld) == 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, v[j], ld);
        const bool desc = ((lane * KPL + j) & size) == 0;
        const uint64_t hi = v[j] > o ? v[j] : o, lo = v[j] > o ? o : v[j];
        v[j] = desc == lower ? hi : lo;
    }
}

template <int KPL>
__device__ __forceinline__ void warp_bitonic_step(uint64_t (&v)[KPL], int size, int d) {
    if (d >= KPL)
        bitonic_across<KPL>(v, size, d);
    else if (d == 1)
        bitonic_in_lane<KPL, 1>(v, size);
    else if (d == 2)
        bitonic_in_lane<KPL, (KPL > 2 ? 2 : 1)>(v, size);  // (d == 2 only when KPL > 2)
    else
        bitonic_in_lane<KPL, (KPL > 4 ? 4 : 1)>(v, size);  // (d == 4 only when KPL > 4)
}

// The loops over the network's stages stay rolled: these kernels run once per
// search on a few SMs, often with their code evicted from L2, and a fully
// unrolled network is tens of KB of straight-line code to fetch.

// Sort the warp's 32 * KPL keys descending.
template <int KPL>
__device__ __forceinline__ void warp_sort_list(uint64_t (&v)[KPL]) {
#pragma unroll 1
    for (int size = 2; size <= 32 * KPL; size <<= 1) {
#pragma unroll 1
        for (int d = size >> 1; d > 0; d >>= 1) warp_bitonic_step<KPL>(v, size, d);
    }
}

// a <- the best 32 * KPL keys of a and b (both sorted descending), sorted descending.
template <int KPL>
__device__ __forceinline__ void warp_fold_list(uint64_t (&a)[KPL], const uint64_t (&b)[KPL]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const uint64_t o = __shfl_sync(0xFFFFFFFFu, b[KPL - 1 - j], 31 - lane);  // b[N - 1 - e]
        a[j] = a[j] > o ? a[j] : o;
    }
#pragma unroll 1
    for (int d = 16 * KPL; d > 0; d >>= 1) warp_bitonic_step<KPL>(a, 64 * KPL, d);  // all descending
}

template <int KPL>
__device__ __noinline__ void block_top_sorted_impl(const uint64_t* keys, int n, K4Smem& sm) {
    constexpr int N = 32 * KPL;
    constexpr int W = K4_THREADS / 32;
    static_assert(W * N <= K4_SORT_MAX, "the warps' lists are folded in sm.sorted");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t a[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) a[j] = KEY_MIN;
    for (int base = warp * N; base < n; base += W * N) {
        uint64_t b[KPL];
        bool any = false;
        const uint64_t least = __shfl_sync(0xFFFFFFFFu, a[KPL - 1], 31);  // the list's last key
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
            const int i = base + j * 32 + lane;  // coalesced; the order within a chunk is irrelevant
            b[j] = i < n ? keys[i] : KEY_MIN;
            any |= b[j] > least;
        }
        if (!__any_sync(0xFFFFFFFFu, any)) continue;  // nothing here enters the list
        warp_sort_list<KPL>(b);
        warp_fold_list<KPL>(a, b);
    }
    __syncthreads();  // callers may still read sm.sorted before this call
#pragma unroll
    for (int j = 0; j < KPL; ++j) sm.sorted[warp * N + lane * KPL + j] = a[j];
    __syncthreads();
#pragma unroll
    for (int half = W / 2; half >= 1; half >>= 1) {
        if (warp < half) {
            uint64_t b[KPL];
#pragma unroll
            for (int j = 0; j < KPL; ++j) b[j] = sm.sorted[(warp + half) * N + lane * KPL + j];
            warp_fold_list<KPL>(a, b);
#pragma unroll
            for (int j = 0; j < KPL; ++j) sm.sorted[warp * N + lane * KPL + j] = a[j];
        }
        __syncthreads();
    }
}

// The min(r, n) largest of n keys, sorted descending, in sm.sorted[0 .. r)
// (KEY_MIN past the n-th); 1 <= r <= K4_TOP_MAX. Block-wide.
__device__ inline void block_top_sorted(const uint64_t* keys, int n, int r, K4Smem& sm) {
    if (r <= 32)
        block_top_sorted_impl<1>(keys, n, sm);
    else if (r <= 64)
        block_top_sorted_impl<2>(keys, n, sm);
    else if (r <= 128)
        block_top_sorted_impl<4>(keys, n, sm);
    else
        block_top_sorted_impl<8>(keys, n, sm);
}

// ---------------------------------------------------------------------------
// Bucket select (n <= K4_BUCKET_N keys, r <= K4_BUCKET_R): the keys stay in
// registers (K4_BUCKET_PT per thread); the score part of each key, ord(score),
// is binned linearly over the block's own [min, max] range into K4_BINS bins
// (a monotone map, so a higher bin holds only greater keys). One histogram, a
// suffix scan over the bins and the boundary bin B (the bin holding the r-th
// best key) give every candidate (bin >= B) its place: the keys in higher
// bins, plus the keys of its own bin that beat it. Six block barriers; the
// only comparisons are within a bin. Gives up (returns false, before writing
// any output) when the boundary bin or the candidate set is too large to rank
// this way, e.g. many equal scores.
// ---------------------------------------------------------------------------
constexpr int K4_BUCKET_PT = 16;
constexpr int K4_BUCKET_N = K4_BUCKET_PT * K4_THREADS;  // 4096
constexpr int K4_BUCKET_R = 1024;          // outputs, in sm.sorted[0 .. 1024)
constexpr int K4_BUCKET_M = 1024;          // candidates, held in sm.sorted[1024 ..)
constexpr int K4_BUCKET_BIN_MAX = 256;     // keys in the boundary bin
static_assert(K4_BINS == 8 * K4_THREADS, "each thread owns eight bins in the scan");
static_assert(K4_BUCKET_R + K4_BUCKET_M <= K4_SORT_MAX, "outputs and candidates share sm.sorted");

__device__ __forceinline__ uint32_t bucket_of(uint64_t key, uint32_t lo, float scale) {
    const uint32_t b = (uint32_t)((float)((uint32_t)(key >> 32) - lo) * scale);
    return b < (uint32_t)K4_BINS ? b : (uint32_t)K4_BINS - 1;
}

// The best min(r, valid) keys sorted descending in sm.sorted[0 .. r), KEY_MIN
// after them (KEY_MIN entries of the input are not keys). Block-wide; every
// thread gets the same return value.
__device__ inline bool block_top_bucket(const uint64_t* keys, int n, int r, K4Smem& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int W = K4_THREADS / 32;
    uint64_t kv[K4_BUCKET_PT];
    uint32_t lo = 0xFFFFFFFFu, hi = 0, valid = 0;
#pragma unroll
    for (int j = 0; j < K4_BUCKET_PT; ++j) {
        const int i = tid + j * K4_THREADS;
        kv[j] = i < n ? keys[i] : KEY_MIN;
        if (kv[j] != KEY_MIN) {
            const uint32_t o = (uint32_t)(kv[j] >> 32);
            lo = o < lo ? o : lo;
            hi = o > hi ? o : hi;
            ++valid;
        }
    }
    for (int b = tid; b < K4_BINS; b += K4_THREADS) sm.hist[b] = 0;
    if (tid == 0) sm.n_collected = 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint32_t l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, off), h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
        valid += __shfl_xor_sync(0xFFFFFFFFu, valid, off);
    }
    if (lane == 0) {
        sm.part[warp] = lo;
        sm.part[W + warp] = hi;
        sm.part[2 * W + warp] = valid;
    }
    __syncthreads();  // (1)
    lo = sm.part[0];
    hi = sm.part[W];
    valid = sm.part[2 * W];
#pragma unroll
    for (int w = 1; w < W; ++w) {
        lo = sm.part[w] < lo ? sm.part[w] : lo;
        hi = sm.part[W + w] > hi ? sm.part[W + w] : hi;
        valid += sm.part[2 * W + w];
    }
    const float scale = (float)K4_BINS / ((float)(hi - lo) + 1.0f);
#pragma unroll
    for (int j = 0; j < K4_BUCKET_PT; ++j)
        if (kv[j] != KEY_MIN) atomicAdd(&sm.hist[bucket_of(kv[j], lo, scale)], 1u);
    __syncthreads();  // (2)
    // thread t owns bins [8t, 8t + 8); count the keys in higher bins
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        c[i] = sm.hist[8 * tid + i];
        sum += c[i];
    }
    uint32_t incl = sum;  // suffix sum over the warp's lanes >= lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, off);
        if (lane + off < 32) incl += v;
    }
    if (lane == 0) sm.part[3 * W + warp] = incl;  // the warp's total
    __syncthreads();  // (3)
    uint32_t run = incl - sum;
    for (int w = warp + 1; w < W; ++w) run += sm.part[3 * W + w];
    const uint32_t want = (uint32_t)r < valid ? (uint32_t)r : valid;  // keys to output
    // start of each bin's region (bins in descending order); the boundary bin
#pragma unroll
    for (int i = 7; i >= 0; --i) {
        if (want > 0 && run < want && want <= run + c[i]) {
            sm.found_prefix = (uint64_t)(8 * tid + i);
            sm.found_count = run + c[i];  // candidates: every key in bins >= B
            sm.found_remaining = c[i];
        }
        sm.hist[8 * tid + i] = run;
        run += c[i];
    }
    if (want == 0 && tid == 0) {
        sm.found_prefix = (uint64_t)K4_BINS;  // no candidates
        sm.found_count = 0;
        sm.found_remaining = 0;
    }
    __syncthreads();  // (4)
    const uint32_t B = (uint32_t)sm.found_prefix;
    const uint32_t m = sm.found_count;
    if (m > (uint32_t)K4_BUCKET_M || sm.found_remaining > (uint32_t)K4_BUCKET_BIN_MAX) return false;
    uint64_t* cand = sm.sorted + K4_BUCKET_R;
#pragma unroll
    for (int j = 0; j < K4_BUCKET_PT; ++j) {
        if (kv[j] == KEY_MIN) continue;
        const uint32_t b = bucket_of(kv[j], lo, scale);
        if (b >= B) cand[atomicAdd(&sm.hist[b], 1u)] = kv[j];
    }
    __syncthreads();  // (5)
    // sm.hist[b] is now the end of bin b's region, and its start the end of bin b + 1's
    for (uint32_t i = tid; i < m; i += K4_THREADS) {
        const uint64_t key = cand[i];
        const uint32_t b = bucket_of(key, lo, scale);
        const uint32_t start = b + 1 < (uint32_t)K4_BINS ? sm.hist[b + 1] : 0u, end = sm.hist[b];
        uint32_t place = start;
        for (uint32_t p = start; p < end; ++p) place += cand[p] > key;
        if (place < want) sm.sorted[place] = key;
    }
    for (int i = (int)want + tid; i < r; i += K4_THREADS) sm.sorted[i] = KEY_MIN;
    __syncthreads();  // (6)
    return true;
}

// The best r keys sorted descending in sm.sorted[0 .. r) (KEY_MIN after the
// valid ones) by the bucket select, or by the register top-r where that gives
// up; false (nothing written) when neither applies. Block-wide.
__device__ inline bool block_top(const uint64_t* keys, int n, int r, K4Smem& sm) {
    if (r <= K4_BUCKET_R && n <= K4_BUCKET_N && block_top_bucket(keys, n, r, sm)) return true;
    if (r > K4_TOP_MAX) return false;
    block_top_sorted(keys, n, r, sm);
    return true;
}

// Keys with this prefix, appended to sm.sorted (warp-aggregated: one
// shared-memory atomic per warp and pass). Block-wide; returns their number.
__device__ __forceinline__ uint32_t gather_prefix(const uint64_t* keys, int n, uint64_t mask, uint64_t prefix,
                                                  K4Smem& sm) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) sm.n_collected = 0;
    __syncthreads();
    for (int base = 0; base < n; base += K4_THREADS) {
        const int i = base + threadIdx.x;
        uint64_t key = 0;
        bool in = false;
        if (i < n) {
            key = keys[i];
            in = (key & mask) == prefix;
        }
        const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, in);
        if (ballot) {
            const int leader = __ffs(ballot) - 1;
            uint32_t slot0 = 0;
            if (lane == leader) slot0 = atomicAdd(&sm.n_collected, (uint32_t)__popc(ballot));
            slot0 = __shfl_sync(0xFFFFFFFFu, slot0, leader);
            if (in) sm.sorted[slot0 + __popc(ballot & lanemask_lt())] = key;
        }
    }
    __syncthreads();
    return sm.n_collected;
}

// r-th largest of the `count` keys in sm.sorted (1-based, counting repeats),
// by counting; count <= K4_THREADS. Block-wide.
__device__ __forceinline__ uint64_t rank_select(uint32_t count, uint32_t r, K4Smem& sm) {
    const int tid = threadIdx.x;
    if (tid < (int)count) {
        const uint64_t mine = sm.sorted[tid];
        uint32_t above_me = 0, equal = 0;
        for (uint32_t j = 0; j < count; ++j) {
            above_me += sm.sorted[j] > mine;
            equal += sm.sorted[j] == mine;
        }
        if (above_me < r && r <= above_me + equal) sm.result = mine;
    }
    __syncthreads();
    const uint64_t res = sm.result;
    __syncthreads();  // callers may reuse sm.sorted and sm.result at once
    return res;
}

// r-th largest (1-based, counting repeats) of n keys; 1 <= r <= n. Block-wide.
// Lists of at most K4_THREADS keys are ranked directly. Otherwise the bits
// all keys share (from the block's minimum and maximum) are skipped, and
// radix passes over the remaining bits, most significant digit first (11 bits
// at a time, a 2048-bin shared-memory histogram), narrow the candidates to a
// prefix until at most K4_THREADS keys share it; those are ranked directly.
// Kept keys cluster (they are the best scores of one query), so histogram
// increments are combined per warp for lanes that hit the same bin.
__device__ inline uint64_t block_kth_largest(const uint64_t* keys, int n, int r, K4Smem& sm) {
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    if (block_top(keys, n, r, sm)) {
        const uint64_t res = sm.sorted[r - 1];
        __syncthreads();  // callers may reuse sm.sorted at once
        return res;
    }
    if (n <= K4_THREADS) return rank_select(gather_prefix(keys, n, 0ull, 0ull, sm), (uint32_t)r, sm);
    // bits common to every key
    uint64_t lo = ~0ull, hi = 0ull;
    for (int i = tid; i < n; i += K4_THREADS) {
        const uint64_t key = keys[i];
        lo = key < lo ? key : lo;
        hi = key > hi ? key : hi;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, off), h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
    }
    if (lane == 0) {
        sm.sorted[warp] = lo;
        sm.sorted[K4_THREADS / 32 + warp] = hi;
    }
    __syncthreads();
    lo = sm.sorted[0];
    hi = sm.sorted[K4_THREADS / 32];
    for (int w = 1; w < K4_THREADS / 32; ++w) {
        lo = sm.sorted[w] < lo ? sm.sorted[w] : lo;
        hi = sm.sorted[K4_THREADS / 32 + w] > hi ? sm.sorted[K4_THREADS / 32 + w] : hi;
    }
    __syncthreads();
    if (lo == hi) return lo;  // every key equal
    int shift = 64 - __clzll((long long)(lo ^ hi));  // bits [shift, 64) are common
    uint64_t mask = shift >= 64 ? 0ull : ~((1ull << shift) - 1ull);
    uint64_t prefix = hi & mask;
    uint32_t remaining = (uint32_t)r;
#pragma unroll 1
    while (shift > 0) {
        const int w = shift >= 11 ? 11 : shift;
        shift -= w;
        const int nb = 1 << w;
        const int per = (nb + K4_THREADS - 1) / K4_THREADS;  // bins thread t sums: [t*per, t*per + per)
        for (int i = tid; i < nb; i += K4_THREADS) sm.hist[i] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += K4_THREADS) {
            const int i = base + tid;
            bool in = false;
            uint32_t bin = 0;
            if (i < n) {
                const uint64_t key = keys[i];
                in = (key & mask) == prefix;
                bin = (uint32_t)(key >> shift) & (uint32_t)(nb - 1);
            }
            // lanes outside the prefix get tags no other lane has
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, in ? bin : (0x80000000u | (uint32_t)lane));
            if (in && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], (uint32_t)__popc(peers));
        }
        __syncthreads();
        // Thread t owns bins [t*per, (t+1)*per); above[t] = count in higher bins.
        uint32_t local = 0;
        for (int i = 0; i < per; ++i)
            if (tid * per + i < nb) local += sm.hist[tid * per + i];
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
        if (local > 0 && above < remaining && remaining <= above + local) {
            uint32_t run = above;
            for (int i = per - 1; i >= 0; --i) {
                if (tid * per + i >= nb) continue;
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
        if (count <= (uint32_t)K4_THREADS) return rank_select(gather_prefix(keys, n, mask, prefix, sm), remaining, sm);
    }
    return prefix;
}

// Keys greater than `th`, appended to sm.sorted (warp-aggregated), at most
// `limit` of them stored. Block-wide; returns their number (may exceed limit).
__device__ __forceinline__ uint32_t gather_above(const uint64_t* keys, int n, uint64_t th, uint32_t limit,
                                                 K4Smem& sm) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) sm.n_collected = 0;
    __syncthreads();
    for (int base = 0; base < n; base += K4_THREADS) {
        const int i = base + threadIdx.x;
        uint64_t key = 0;
        bool in = false;
        if (i < n) {
            key = keys[i];
            in = key > th;
        }
        const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, in);
        if (ballot) {
            const int leader = __ffs(ballot) - 1;
            uint32_t slot0 = 0;
            if (lane == leader) slot0 = atomicAdd(&sm.n_collected, (uint32_t)__popc(ballot));
            slot0 = __shfl_sync(0xFFFFFFFFu, slot0, leader);
            const uint32_t slot = slot0 + __popc(ballot & lanemask_lt());
            if (in && slot < limit) sm.sorted[slot] = key;
        }
    }
    __syncthreads();
    return sm.n_collected;
}

// The min(n_valid, k) largest of n keys, sorted descending, written as
// (id, score); slots past n_valid get (-1, -inf). The keys are distinct
// except for KEY_MIN entries (empty slots), and n_valid of them are not
// KEY_MIN. Block-wide; out_* point at one list's row of k entries.
__device__ inline void write_sorted_topk(const uint64_t* keys, int n, int n_valid, int k, K4Smem& sm,
                                         int32_t* out_ids, float* out_scores) {
    const int tid = threadIdx.x;
    const int r = n_valid < k ? n_valid : k;
    for (int i = r + tid; i < k; i += K4_THREADS) {
        out_ids[i] = -1;
        out_scores[i] = -INFINITY;
    }
    if (r == 0) return;
    if (block_top(keys, n, r, sm)) {
        for (int i = tid; i < r; i += K4_THREADS) {
            out_ids[i] = (int32_t)key_id(sm.sorted[i]);
            out_scores[i] = key_score(sm.sorted[i]);
        }
        __syncthreads();
        return;
    }
    const uint64_t kth = block_kth_largest(keys, n, r, sm);
    // the r best: the keys above the r-th largest (r - 1 of them when keys
    // are distinct), then the r-th largest in the remaining slots
    uint32_t above = gather_above(keys, n, kth, (uint32_t)r, sm);
    if (above > (uint32_t)r) above = (uint32_t)r;
    for (int i = (int)above + tid; i < r; i += K4_THREADS) sm.sorted[i] = kth;
    __syncthreads();
    if (r <= 2 * K4_THREADS) {
        // sort by rank: a key's place is the number of keys above it
        for (int i = tid; i < r; i += K4_THREADS) {
            const uint64_t mine = sm.sorted[i];
            int place = 0;
            for (int j = 0; j < r; ++j) place += sm.sorted[j] > mine || (sm.sorted[j] == mine && j < i);
            out_ids[place] = (int32_t)key_id(mine);
            out_scores[place] = key_score(mine);
        }
        __syncthreads();
        return;
    }
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
    for (int i = tid; i < r; i += K4_THREADS) {
        out_ids[i] = (int32_t)key_id(sm.sorted[i]);
        out_scores[i] = key_score(sm.sorted[i]);
    }
    __syncthreads();
}

}  // namespace tt
