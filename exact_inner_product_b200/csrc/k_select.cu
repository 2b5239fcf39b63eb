// k_select.cu - K4: per-query selection over the candidate keys kept by a
// scoring pass, plus the small bookkeeping kernels.
//
// One CTA per query; the kept keys are staged in shared memory when they fit.
// The r-th largest key is found by a most-significant-digit radix select over
// the 64-bit keys (digits of 11/11/10/11/11/10 bits, a 2048-bin shared-memory
// histogram per digit) until at most 256 keys share the selected prefix;
// those are ranked directly. Its cost depends only on the number of kept
// keys, not on how they are ordered. Keys are
// distinct (the low word encodes the candidate id), so exactly r keys are
// >= the r-th largest.
//
// Threshold mode: the next level's filter key is (r-th largest) - 1, so a
// later pass keeps every key >= it.
// Final mode: the kept keys >= the k-th largest are gathered, sorted
// descending with a shared-memory bitonic sort and written as (id, score);
// positions past the number of eligible candidates get (-1, -inf). The
// result is exact when the pass kept every key above its threshold
// (count <= cap) and either found at least k of them or had no threshold;
// otherwise the list is handed to the exact fallback scan (k_exact.cu),
// which runs in the same stream right after, with no host involvement.
// (Order: score descending, ties by ascending id - mhtirogla.ai Two-tower
// retrieval, Code, Towers::top_k; padding replaces the bf16.min fill of
// recsys_two_tower_model.py `mask_and_top_k`.)
#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"
#include "tt_select.cuh"

namespace tt {
namespace {

// Merge of per-shard results: part p holds, for every query, its shard's
// top-k_in as (local id, score); local ids plus id_offset[p] are global ids;
// -1 entries are padding. Each query's keys are built in shared memory (or
// in scratch[q * parts * k_in ...] when they do not fit) and the k_out best
// are written sorted. Exact: every member of the global top-k_out is in its
// own shard's top-k_in when k_out <= k_in.
struct MergeOffsets {
    int64_t v[TT_MAX_PARTS];
};

__global__ void __launch_bounds__(K4_THREADS)
    k4_merge(const int32_t* __restrict__ ids, const float* __restrict__ scores, int parts, int b, int k_in,
             const MergeOffsets id_offset, int k_out, uint64_t* __restrict__ scratch,
             int32_t* __restrict__ out_ids, float* __restrict__ out_scores) {
    extern __shared__ __align__(16) uint8_t k4_smem_raw[];
    K4Smem& sm = *reinterpret_cast<K4Smem*>(k4_smem_raw);
    const int q = blockIdx.x;
    const int tid = threadIdx.x;
    const int m = parts * k_in;
    uint64_t* keys = m <= K4_SMEM_KEYS ? sm.keys : scratch + (int64_t)q * m;
    if (tid == 0) sm.n_collected = 0;
    __syncthreads();
    for (int i = tid; i < m; i += K4_THREADS) {
        const int p = i / k_in, j = i - p * k_in;
        const int64_t src = ((int64_t)p * b + q) * k_in + j;
        const int32_t id = ids[src];
        if (id >= 0) keys[atomicAdd(&sm.n_collected, 1u)] = make_key(scores[src], (uint32_t)(id + id_offset.v[p]));
    }
    __syncthreads();
    const int n = (int)sm.n_collected;
    __syncthreads();
    write_sorted_topk(keys, n, n, k_out, sm, out_ids + (int64_t)q * k_out, out_scores + (int64_t)q * k_out);
}

__global__ void __launch_bounds__(K4_THREADS)
    k4_select_threshold(const uint64_t* __restrict__ keys, uint32_t* __restrict__ count, int cap,
                        int r, uint64_t* __restrict__ theta_next, float* __restrict__ thf_next) {
    extern __shared__ __align__(16) uint8_t k4_smem_raw[];
    K4Smem& sm = *reinterpret_cast<K4Smem*>(k4_smem_raw);
    pdl_trigger();
    pdl_wait();  // the pass that kept the keys is done
    const int q = blockIdx.x;
    const uint32_t c = count[q];
    const int n = c < (uint32_t)cap ? (int)c : cap;
    uint64_t th = KEY_MIN;
    if (n >= r && r > 0) {
        // the register top-r reads every key once: no staging for it
        const uint64_t* qkeys = r <= K4_TOP_MAX ? keys + (int64_t)q * cap : stage_keys(keys + (int64_t)q * cap, n, sm);
        th = block_kth_largest(qkeys, n, r, sm) - 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        theta_next[q] = th;
        thf_next[q] = key_floor(th);
        count[q] = 0;
    }
}

// Final mode. A list whose pass kept everything above its threshold is
// exact: its sorted top-k is written. Otherwise it is handed to the exact
// fallback scan (k_exact.cu): its index goes to flagged[atomicAdd(flags[0])]
// and theta[q] receives a valid lower bound on its true k-th best key (the
// k-th best kept key minus one after an overflow, else KEY_MIN).
__global__ void __launch_bounds__(K4_THREADS)
    k4_select_final(const uint64_t* __restrict__ keys, uint32_t* __restrict__ count, int cap, int k,
                    uint64_t* __restrict__ theta, float* __restrict__ thf, int32_t* __restrict__ flagged,
                    int* __restrict__ flags, int32_t* __restrict__ out_ids, float* __restrict__ out_scores) {
    extern __shared__ __align__(16) uint8_t k4_smem_raw[];
    K4Smem& sm = *reinterpret_cast<K4Smem*>(k4_smem_raw);
    pdl_trigger();
    pdl_wait();  // the pass that kept the keys is done
    const int q = blockIdx.x;
    const int tid = threadIdx.x;
    if (flags[1] != 0) return;  // a device wait expired earlier in this call: nothing is valid
    const uint32_t c = count[q];
    const int n = c < (uint32_t)cap ? (int)c : cap;
    const uint64_t th = theta[q];
    const uint64_t* qkeys = k <= K4_TOP_MAX ? keys + (int64_t)q * cap : stage_keys(keys + (int64_t)q * cap, n, sm);
    const bool exact = (c <= (uint32_t)cap) && (c >= (uint32_t)k || th == KEY_MIN);
    if (exact) {
        write_sorted_topk(qkeys, n, n, k, sm, out_ids + (int64_t)q * k, out_scores + (int64_t)q * k);
    } else {
        // After an overflow every key above th survived, and n >= k of them
        // were kept: the k-th best kept key is at most the true k-th best.
        uint64_t th_new = KEY_MIN;
        if (c > (uint32_t)cap && n >= k) th_new = block_kth_largest(qkeys, n, k, sm) - 1;
        if (tid == 0) {
            theta[q] = th_new;
            thf[q] = key_floor(th_new);
            flagged[atomicAdd(flags, 1)] = q;
        }
    }
    __syncthreads();
    if (tid == 0) count[q] = 0;
}

__global__ void k4_init(uint32_t* count, uint64_t* theta, float* thf, uint64_t th0, int b, int b_pad,
                        int* flags) {
    pdl_trigger();
    pdl_wait();  // the previous search on this work memory is done with it
    const float f0 = key_floor(th0), fmax = key_floor(KEY_MAX);
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < b_pad; q += gridDim.x * blockDim.x) {
        if (q < b) {
            count[q] = 0;
            theta[q] = th0;
            thf[q] = f0;
        } else {
            theta[q] = KEY_MAX;
            thf[q] = fmax;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < 16) flags[threadIdx.x] = 0;
}

__global__ void k4_pad(int32_t* out_ids, float* out_scores, int64_t count) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
         i += (int64_t)gridDim.x * blockDim.x) {
        out_ids[i] = -1;
        out_scores[i] = -INFINITY;
    }
}

// Exclusion words of rows [start, start + count): bit i of out word w is bit
// (start + 32w + i) of the input mask (0 past the end, or when there is no
// input mask). With `types`, a row whose type differs from `want` is
// excluded as well.
__global__ void k4_mask_slice(const uint32_t* __restrict__ in, int64_t start, int64_t count,
                              const uint8_t* __restrict__ types, int want, uint32_t* __restrict__ out) {
    const int64_t words = (count + 31) / 32;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (int64_t)gridDim.x * blockDim.x) {
        uint32_t v = 0;
        for (int i = 0; i < 32; ++i) {
            const int64_t r = 32 * w + i;
            if (r >= count) break;
            const int64_t j = start + r;
            bool ex = in != nullptr && ((in[j >> 5] >> (j & 31)) & 1u);
            if (types != nullptr && types[j] != (uint8_t)want) ex = true;
            v |= (ex ? 1u : 0u) << i;
        }
        out[w] = v;
    }
}

// ids += offset where ids >= 0 (padding stays -1).
__global__ void k4_offset_ids(int32_t* ids, int64_t count, int64_t offset) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t v = ids[i];
        if (v >= 0) ids[i] = (int32_t)(v + offset);
    }
}

unsigned small_grid(int64_t n) {
    int64_t g = (n + 255) / 256;
    if (g < 1) g = 1;
    if (g > 1024) g = 1024;
    return (unsigned)g;
}

}  // namespace

cudaError_t launch_init(uint32_t* count, uint64_t* theta, float* thf, uint64_t theta_value, int b,
                        int b_pad, int* flags, cudaStream_t s) {
    note_launch_begin(TT_KIND_AUX, s);
    const cudaError_t e = launch_pdl(k4_init, dim3(small_grid(b_pad)), dim3(256), 0, s, count, theta, thf,
                                     theta_value, b, b_pad, flags);
    note_launch_end(TT_KIND_AUX, s);
    return e;
}

cudaError_t launch_select_threshold(const uint64_t* keys, uint32_t* count, int cap, int b, int r,
                                    uint64_t* theta_next, float* thf_next, cudaStream_t s) {
    if (b == 0) return cudaSuccess;
    const int smem = (int)sizeof(K4Smem);
    cudaFuncSetAttribute(k4_select_threshold, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch_begin(TT_KIND_SELECT, s);
    const cudaError_t e = launch_pdl(k4_select_threshold, dim3(b), dim3(K4_THREADS), smem, s, keys, count, cap, r,
                                     theta_next, thf_next);
    note_launch_end(TT_KIND_SELECT, s);
    return e;
}

cudaError_t launch_select_final(const uint64_t* keys, uint32_t* count, int cap, int b, int k,
                                uint64_t* theta, float* thf, int32_t* flagged, int* flags,
                                int32_t* out_ids, float* out_scores, cudaStream_t s) {
    if (b == 0) return cudaSuccess;
    const int smem = (int)sizeof(K4Smem);
    cudaFuncSetAttribute(k4_select_final, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch_begin(TT_KIND_SELECT, s);
    const cudaError_t e = launch_pdl(k4_select_final, dim3(b), dim3(K4_THREADS), smem, s, keys, count, cap, k,
                                     theta, thf, flagged, flags, out_ids, out_scores);
    note_launch_end(TT_KIND_SELECT, s);
    return e;
}

cudaError_t launch_merge(const int32_t* ids, const float* scores, int parts, int b, int k_in,
                         const int64_t* id_offset_host, int k_out, uint64_t* scratch, int32_t* out_ids,
                         float* out_scores, cudaStream_t s) {
    if (b == 0) return cudaSuccess;
    if (parts < 1 || parts > TT_MAX_PARTS) return cudaErrorInvalidValue;
    MergeOffsets id_offset;
    for (int p = 0; p < TT_MAX_PARTS; ++p) id_offset.v[p] = p < parts ? id_offset_host[p] : 0;
    const int smem = (int)sizeof(K4Smem);
    cudaFuncSetAttribute(k4_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    note_launch_begin(TT_KIND_SELECT, s);
    k4_merge<<<b, K4_THREADS, smem, s>>>(ids, scores, parts, b, k_in, id_offset, k_out, scratch, out_ids,
                                         out_scores);
    note_launch_end(TT_KIND_SELECT, s);
    return cudaGetLastError();
}

int merge_smem_keys() { return K4_SMEM_KEYS; }

cudaError_t launch_mask_slice(const uint32_t* in, int64_t start, int64_t count, const uint8_t* types, int want,
                              uint32_t* out, cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    note_launch_begin(TT_KIND_AUX, s);
    k4_mask_slice<<<small_grid((count + 31) / 32), 256, 0, s>>>(in, start, count, types, want, out);
    note_launch_end(TT_KIND_AUX, s);
    return cudaGetLastError();
}

cudaError_t launch_offset_ids(int32_t* ids, int64_t count, int64_t offset, cudaStream_t s) {
    if (count == 0 || offset == 0) return cudaSuccess;
    note_launch_begin(TT_KIND_AUX, s);
    k4_offset_ids<<<small_grid(count), 256, 0, s>>>(ids, count, offset);
    note_launch_end(TT_KIND_AUX, s);
    return cudaGetLastError();
}

cudaError_t launch_pad(int32_t* out_ids, float* out_scores, int64_t count, cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    note_launch_begin(TT_KIND_AUX, s);
    k4_pad<<<small_grid(count), 256, 0, s>>>(out_ids, out_scores, count);
    note_launch_end(TT_KIND_AUX, s);
    return cudaGetLastError();
}

// Per query: the loosest of its sets' thresholds, which every kernel's first
// test uses before the exact per-set test.
__global__ void k4_sets_min(const uint64_t* __restrict__ theta_v, const float* __restrict__ thf_v, int n_sets,
                            int b, int b_pad, uint64_t* __restrict__ theta_min, float* __restrict__ thf_min) {
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= b_pad) return;
    uint64_t t = KEY_MAX;
    float f = key_floor(KEY_MAX);
    if (q < b) {
        for (int s = 0; s < n_sets; ++s) {
            const uint64_t ts = theta_v[(int64_t)s * b + q];
            if (ts < t) t = ts;
            f = fminf(f, thf_v[(int64_t)s * b + q]);
        }
    }
    theta_min[q] = t;
    thf_min[q] = f;
}

cudaError_t launch_sets_min(const uint64_t* theta_v, const float* thf_v, int n_sets, int b, int b_pad,
                            uint64_t* theta_min, float* thf_min, cudaStream_t s) {
    if (b_pad <= 0) return cudaSuccess;
    note_launch_begin(TT_KIND_AUX, s);
    k4_sets_min<<<(b_pad + 255) / 256, 256, 0, s>>>(theta_v, thf_v, n_sets, b, b_pad, theta_min, thf_min);
    note_launch_end(TT_KIND_AUX, s);
    return cudaGetLastError();
}

}  // namespace tt
