// k_exact.cu - the exact fallback of a search: one launch at the end of every
// tt_score_topk that recomputes, from scratch and without any capacity limit,
// the lists whose filtered pass could not prove its result exact.
//
// The filtered passes keep only candidates whose key beats an estimated
// threshold, in a buffer of `cap` keys per list. The final select proves a
// list exact (nothing above the threshold was dropped, and at least k keys,
// or every eligible key, were kept); a list it cannot prove is appended to
// `flagged`, with a valid lower bound on its true k-th best key in theta
// (after an overflow: the k-th best kept key minus one; otherwise KEY_MIN).
// This kernel then runs in the same stream, so a search never needs the host
// to look at the result: when nothing is flagged (the common case) every
// block returns at once.
//
// Work units are (flagged list, corpus chunk). A block scans its chunk one row
// per thread, scoring with the same arithmetic as the streaming scorer (an
// fp32 fused multiply-add chain over the row in element order, then one
// multiply by c_j = fl(inv_norm_j * fl(1/tau)); int8 rows: the exact int32
// code sum, then fl(fl(acc * us) * c_j)), and keeps every key above a running
// block threshold in shared memory. When the buffer fills up it keeps only
// the k best and raises the threshold to the k-th best minus one, so the
// chunk's exact top-k is all that remains at the end. The block that finishes
// a list's last chunk merges the chunks' lists into the final sorted top-k.
// (On the tensor-core paths the main passes sum products on the tensor cores;
// a list recomputed here can differ from them in the last bit of a score.)
//
// If a bounded wait of an earlier kernel of the call expired (flags[1] != 0)
// nothing is valid: every output entry becomes (id -1, score NaN).
// The status block (host-mapped memory of the index handle, when given)
// receives the error code (only when there is one), the number of lists
// recomputed here and the call's sequence number.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"
#include "tt_rowdot.cuh"
#include "tt_select.cuh"

namespace tt {
namespace {

constexpr int KX_THREADS = K4_THREADS;
constexpr int KX_BUF = K4_SMEM_KEYS;  // keys a block keeps between compactions

__device__ __forceinline__ int ld_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Keep the k best of the block's n buffered keys (n > k): they move to the
// front of the buffer; returns the k-th best.
__device__ uint64_t compact_to_k(K4Smem& sm, int n, int k, uint32_t* s_count) {
    const uint64_t kth = block_kth_largest(sm.keys, n, k, sm);
    gather_above(sm.keys, n, kth - 1, (uint32_t)k, sm);  // exactly k (keys are distinct and above KEY_MIN)
    for (int i = threadIdx.x; i < k; i += KX_THREADS) sm.keys[i] = sm.sorted[i];
    if (threadIdx.x == 0) *s_count = (uint32_t)k;
    __syncthreads();
    return kth;
}

__global__ void __launch_bounds__(KX_THREADS) k4_exact(const ExactArgs a) {
    extern __shared__ __align__(16) uint8_t kx_smem_raw[];
    K4Smem& sm = *reinterpret_cast<K4Smem*>(kx_smem_raw);
    float* qf = reinterpret_cast<float*>(kx_smem_raw + sizeof(K4Smem));  // [d] fp32, or [d/4] code words
    __shared__ uint32_t s_count;
    __shared__ uint64_t s_th;
    __shared__ int s_last;
    const int tid = threadIdx.x;
    pdl_wait();  // launched behind the final select
    const int err = ld_volatile(a.flags + 1);
    const int n_flagged = ld_volatile(a.flags);
    if (blockIdx.x == 0 && tid == 0 && a.status != nullptr) {
        if (err != 0) {
            a.status->err = err;
            __threadfence_system();  // the error is visible no later than the sequence number
        }
        a.status->seq_repaired = ((uint64_t)(uint32_t)a.seq << 32) | (uint32_t)(err != 0 ? 0 : n_flagged);
    }
    if (err != 0) {
        const int64_t total = (int64_t)a.V * a.k;
        for (int64_t i = (int64_t)blockIdx.x * KX_THREADS + tid; i < total; i += (int64_t)gridDim.x * KX_THREADS) {
            a.out_ids[i] = -1;
            a.out_scores[i] = __int_as_float(0x7FC00000);  // NaN
        }
        return;
    }
    if (n_flagged == 0) return;

    const int C = a.chunks;
    const int k = a.k;
    const int d = a.d;
    const int64_t units = (int64_t)n_flagged * C;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int f = (int)(u / C);
        const int c = (int)(u - (int64_t)f * C);
        const int v = a.flagged[f];
        const int q = v % a.b;
        const int set = v / a.b;
        // the list's query, as the main passes saw it
        __syncthreads();  // the previous unit is done with qf and the buffer
        stage_query(a.dtype, a.queries, a.q_dtype, q, d, qf);
        if (tid == 0) {
            s_count = 0;
            s_th = a.theta[v];
        }
        __syncthreads();
        const float us = a.dtype == TT_I8 ? a.qscale[q] : 1.0f;
        const int64_t r0 = a.n * c / C, r1 = a.n * (c + 1) / C;
        for (int64_t base = r0; base < r1; base += KX_THREADS) {
            const uint64_t th = s_th;
            const int64_t r = base + tid;
            if (r < r1) {
                bool ok = true;
                if (a.exclude) ok = !((a.exclude[r >> 5] >> (r & 31)) & 1u);
                if (ok && a.types) ok = a.set_of[a.types[r]] == set;
                if (ok) {
                    const float s = score_row(a.dtype, a.rows, r, d, qf, a.inv_norm, a.inv_tau, us);
                    const uint64_t key = make_key(s, (uint32_t)r);
                    if (key > th) sm.keys[atomicAdd(&s_count, 1u)] = key;
                }
            }
            __syncthreads();
            const uint32_t cnt = s_count;
            if (cnt > (uint32_t)(KX_BUF - KX_THREADS)) {  // block-uniform
                const uint64_t kth = compact_to_k(sm, (int)cnt, k, &s_count);
                if (tid == 0 && kth - 1 > s_th) s_th = kth - 1;
                __syncthreads();
            }
        }
        // this chunk's exact top-k (fewer when the chunk has fewer eligible rows)
        int n = (int)s_count;
        if (n > k) {
            compact_to_k(sm, n, k, &s_count);
            n = k;
        }
        uint64_t* out = a.keys + (int64_t)v * a.cap + (int64_t)c * k;
        for (int i = tid; i < k; i += KX_THREADS) out[i] = i < n ? sm.keys[i] : KEY_MIN;
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(a.done + v, 1u) == (uint32_t)(C - 1);
        __syncthreads();
        if (!s_last) continue;
        // the last chunk of list v: merge the C lists of k keys (C * k <= KX_BUF)
        __threadfence();
        const uint64_t* lk = a.keys + (int64_t)v * a.cap;
        const int m = C * k;
        if (tid == 0) sm.n_collected = 0;
        __syncthreads();
        uint32_t mine = 0;
        for (int i = tid; i < m; i += KX_THREADS) {
            const uint64_t key = __ldcg(lk + i);
            sm.keys[i] = key;
            mine += key != KEY_MIN;
        }
        atomicAdd(&sm.n_collected, mine);
        __syncthreads();
        const int n_valid = (int)sm.n_collected;
        __syncthreads();
        write_sorted_topk(sm.keys, m, n_valid, k, sm, a.out_ids + (int64_t)v * k, a.out_scores + (int64_t)v * k);
    }
}

}  // namespace

int exact_chunks(int64_t n, int k, int cap) {
    int lim = cap < KX_BUF ? cap : KX_BUF;
    int c = lim / k;
    const int64_t by_rows = (n + KX_THREADS - 1) / KX_THREADS;  // at least a block's worth of rows per chunk
    if (c > by_rows) c = (int)by_rows;
    return c < 1 ? 1 : c;
}

cudaError_t launch_exact(const ExactArgs& a, cudaStream_t s, int sm_count) {
    if (a.V == 0 || a.k == 0) return cudaSuccess;
    const size_t smem = sizeof(K4Smem) + (size_t)a.d * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k4_exact, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // one block per SM at most: a search that needs no repair launches few
    // blocks, each of which returns at once
    int64_t grid = (int64_t)a.V * a.chunks;
    const int64_t max_grid = sm_count;
    if (grid > max_grid) grid = max_grid;
    if (grid < 1) grid = 1;
    note_launch_begin(TT_KIND_AUX, s);
    e = launch_pdl(k4_exact, dim3((unsigned)grid), dim3(KX_THREADS), smem, s, a);
    note_launch_end(TT_KIND_AUX, s);
    return e;
}

}  // namespace tt
