// k_estimate.cu - the filter threshold of a small batch (b <= 8 queries on
// the streaming scorer) from one sample of the corpus, in a single launch.
//
// The search keeps, per query, only candidates whose key beats a threshold
// key theta; the r-th best key of a 1/S sample of the rows, minus one, puts
// about r * S candidates of the whole corpus above theta (see the scan plan
// in tt_api.cu, which picks S and r). For a large batch the sample is one
// more filtered pass followed by a select; for a small batch that chain is
// dominated by its launches, so here the sample is scored and reduced to the
// threshold in one kernel:
//   - block (g, q) scores sample rows g*256 .. g*256 + 255, one per thread
//     (level row j is corpus row j * stride), against query q with the same
//     arithmetic as the streaming scorer, and writes its best `rank` keys,
//     sorted (a bitonic top-r in registers), to the query's work buffer;
//   - the last block of query q to finish merges the blocks' lists: their
//     union holds the query's `rank` best sample keys, and the rank-th of
//     them, minus one, is theta[q] (KEY_MIN when fewer keys were eligible).
// (recsys_two_tower_model.py `forward`: scores = user . post_embeddings^T;
// the sample and its rank only decide which candidates the pass keeps, and
// the final select checks that nothing of the true top-k was dropped.)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"
#include "tt_rowdot.cuh"
#include "tt_select.cuh"

namespace tt {
namespace {

constexpr int KE_THREADS = K4_THREADS;
constexpr int KE_ROWS = ESTIMATE_BLOCK_ROWS;  // sample rows per block (<= K4_SMEM_KEYS)
static_assert(KE_ROWS == KE_THREADS, "one sample row per thread");
static_assert(ESTIMATE_MAX_RANK <= K4_TOP_MAX, "a block's best keys are kept in registers");

__global__ void __launch_bounds__(KE_THREADS) k2_estimate(const EstimateArgs a) {
    extern __shared__ __align__(16) uint8_t ke_smem_raw[];
    K4Smem& sm = *reinterpret_cast<K4Smem*>(ke_smem_raw);
    float* qf = reinterpret_cast<float*>(ke_smem_raw + sizeof(K4Smem));
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int g = blockIdx.x, q = blockIdx.y;
    const int G = gridDim.x;
    const int R = a.rank;
    pdl_trigger();  // the streaming pass may launch and wait behind this kernel
    pdl_wait();     // the queries and the work memory are ready
    if (g == 0 && tid == 0 && a.count != nullptr) a.count[q] = 0;
    if (g == 0 && q == 0 && tid < 4 && a.flags != nullptr) a.flags[tid] = 0;
    stage_query(a.dtype, a.queries, a.q_dtype, q, a.d, qf);
    __syncthreads();
    const float us = a.dtype == TT_I8 ? a.qscale[q] : 1.0f;
    {
        const int64_t j = (int64_t)g * KE_ROWS + tid;  // one sample row per thread
        uint64_t key = KEY_MIN;                        // no row, or an excluded one
        if (j < a.n_sample) {
            const int64_t r = j * a.stride;
            if (!(a.exclude && ((a.exclude[r >> 5] >> (r & 31)) & 1u)))
                key = make_key(score_row(a.dtype, a.rows, r, a.d, qf, a.inv_norm, a.inv_tau, us), (uint32_t)r);
        }
        sm.keys[tid] = key;
    }
    __syncthreads();
    // this block's best R keys, sorted (KEY_MIN past the block's eligible rows)
    uint64_t* out = a.keys + (int64_t)q * a.cap + (int64_t)g * R;
    block_top(sm.keys, KE_ROWS, R, sm);  // R <= K4_TOP_MAX: always decides
    for (int i = tid; i < R; i += KE_THREADS) out[i] = sm.sorted[i];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(a.tickets + q, 1) == G - 1;
    __syncthreads();
    if (!s_last) return;
    // the last block of query q: the rank-th best of the blocks' lists
    __threadfence();
    const uint64_t* lk = a.keys + (int64_t)q * a.cap;
    const int m = G * R;
    for (int i = tid; i < m; i += KE_THREADS) sm.keys[i] = __ldcg(lk + i);
    __syncthreads();
    block_top(sm.keys, m, R, sm);
    const uint64_t kth = sm.sorted[R - 1];  // KEY_MIN when fewer than R rows were eligible
    const uint64_t th = kth == KEY_MIN ? KEY_MIN : kth - 1;
    if (tid == 0) {
        a.theta[q] = th;
        a.thf[q] = key_floor(th);
        a.tickets[q] = 0;  // ready for the next search
    }
}

}  // namespace

cudaError_t launch_estimate(const EstimateArgs& a, cudaStream_t s) {
    if (a.b == 0 || a.n_sample == 0) return cudaSuccess;
    const int G = (int)((a.n_sample + KE_ROWS - 1) / KE_ROWS);
    if (a.rank < 1 || a.rank > ESTIMATE_MAX_RANK) return cudaErrorInvalidValue;
    if ((int64_t)G * a.rank > K4_SMEM_KEYS || (int64_t)G * a.rank > a.cap) return cudaErrorInvalidValue;
    const size_t smem = sizeof(K4Smem) + (size_t)a.d * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k2_estimate, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    note_launch_begin(TT_KIND_ESTIMATE, s);
    e = launch_pdl(k2_estimate, dim3((unsigned)G, (unsigned)a.b), dim3(KE_THREADS), smem, s, a);
    note_launch_end(TT_KIND_ESTIMATE, s);
    return e;
}

}  // namespace tt
