// k_tensor.cu - K3: batched scorer on the 5th-generation tensor cores.
//
// For a batch of queries the scores S = V . U^T form a dense contraction
// (recsys_two_tower_model.py `forward` / `compute_top_k`:
// matmul(user.astype(bf16), post_embeddings.T)). This kernel computes it
// tile by tile with tcgen05 MMAs (bf16 operands in shared memory, fp32
// accumulators in tensor memory) and never writes the score matrix: the
// epilogue reads each accumulator tile from TMEM, applies the per-candidate
// scale and the exclusion mask and keeps only candidates whose key beats the
// query's threshold (the same filter as the streaming scorer).
//
// Layout of one MMA: M = 128 corpus rows (TMEM lanes), N = NQ <= 256
// queries (TMEM columns), K = 16. A query tile (NQ x d, bf16) stays resident
// in shared memory for a whole work unit; corpus tiles stream through a ring
// of stages of one or two 16 KB K chunks (128 rows x 64 elements each,
// 128-byte swizzle; two when d has an even number of chunks). Two TMEM
// accumulators (columns 0 and 256) let the epilogue drain tile t while the
// tensor cores work on tile t + 1.
//
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues MMAs (one thread), warps 2..9 are the epilogue: warp w reads
// TMEM lanes 32*(w%4)..+31 (its 32 corpus rows) and one half of the columns.
//
// Work units: (query tile, corpus chunk) with the query tile varying
// fastest, so the CTAs that run at the same time read the same corpus
// chunks and share them through L2.
//
// Every wait is bounded; on expiry the kernel records an error code,
// waits (bounded) for its own copies and MMAs in flight, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int K3_M = 128;                  // corpus rows per tile
constexpr int K3_ROW_BYTES = 128;          // one 128-byte swizzle row of K per operand row
constexpr int K3_STAGE_BYTES = K3_M * 128; // one K chunk of a corpus tile
constexpr int K3_MAX_STAGES = 12;
constexpr int K3_EPI_WARPS = 8;
constexpr int K3_THREADS = 32 * (2 + K3_EPI_WARPS);
constexpr int K3_TMEM_COLS = 512;
constexpr int K3_ACC_COLS = 256;
constexpr int K3_MAX_NQ = 256;
constexpr int K3_SMEM_BUDGET = 227 * 1024;

constexpr int K3_WARP_COLS = K3_MAX_NQ / 2;  // columns one epilogue warp covers at most

struct K3Ctl {
    uint64_t full[K3_MAX_STAGES];
    uint64_t empty[K3_MAX_STAGES];
    uint64_t qfull, qempty;
    uint64_t tfull[2], tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int skip;
    // per epilogue warp: fast-path thresholds and exact threshold keys of its
    // columns for the current unit (int8 rows: and the query scales)
    alignas(16) float th_fast[K3_EPI_WARPS][K3_WARP_COLS];  // read as float4
    uint64_t th_key[K3_EPI_WARPS][K3_WARP_COLS];
    float q_us[K3_EPI_WARPS][K3_WARP_COLS];
};
static_assert(offsetof(K3Ctl, th_fast) % 16 == 0, "float4 reads of th_fast need 16-byte alignment");

struct K3Params {
    PassArgs a;
    int nq;          // queries per tile (multiple of 32, <= 256)
    int q_tiles;     // ceil(b / nq)
    int kchunks;     // 128-byte chunks of K: ceil(d * element size / 128)
    int kps;         // K chunks per ring stage
    int stages;
    int64_t tiles;   // corpus tiles of 128 rows in this level
    int chunks;      // corpus chunks (units = q_tiles * chunks)
    uint32_t idesc;
};

__device__ __forceinline__ void unit_range(const K3Params& p, int u, int* qt, int64_t* t0,
                                           int64_t* t1) {
    *qt = u % p.q_tiles;
    const int ch = u / p.q_tiles;
    *t0 = p.tiles * ch / p.chunks;
    *t1 = p.tiles * (ch + 1) / p.chunks;
}

// I8: int8 codes (kind::i8, int32 accumulators; recsys_two_tower_model.py
// `compute_top_k_int8`), else bf16 (kind::f16, fp32 accumulators).
template <bool I8, int KPS>
__global__ void __launch_bounds__(K3_THREADS, 1)
    k3_tensor(const __grid_constant__ CUtensorMap tm_rows, const __grid_constant__ CUtensorMap tm_q,
              const K3Params p) {
    constexpr int KC = I8 ? 128 : 64;  // elements per 128-byte row of a chunk
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int q_chunk_bytes = p.nq * 128;
    uint8_t* qsm = smem;                                           // [kchunks][nq x 128 B]
    uint8_t* ring = smem + (size_t)p.kchunks * q_chunk_bytes;      // [stages][16 KB]
    K3Ctl* ctl = reinterpret_cast<K3Ctl*>(ring + (size_t)p.stages * KPS * K3_STAGE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.q_tiles * p.chunks;

    // A bounded wait of an earlier pass of this search expired: nothing that
    // follows is valid, so skip the work (decided once for the whole CTA,
    // before any barrier or tensor memory is set up).
    if (threadIdx.x == 0) ctl->skip = *reinterpret_cast<volatile int*>(p.a.err);
    __syncthreads();
    if (ctl->skip) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->qfull, 1);
        mbar_init(&ctl->qempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], K3_EPI_WARPS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, K3_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int* abort = &ctl->abort;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_rows);
            tma_prefetch_desc(&tm_q);
            uint32_t it = 0;
            int uc = 0, q_issued = -1;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
                int qt;
                int64_t t0, t1;
                unit_range(p, u, &qt, &t0, &t1);
                if (!mbar_wait(&ctl->qempty, (uc & 1) ^ 1, abort)) { ok = false; break; }
                q_issued = uc;
                mbar_arrive_expect_tx(&ctl->qfull, (uint32_t)(p.kchunks * q_chunk_bytes));
                for (int kc = 0; kc < p.kchunks; ++kc)
                    tma_load_2d(qsm + (size_t)kc * q_chunk_bytes, &tm_q, &ctl->qfull, kc * KC,
                                qt * p.nq);
                for (int64_t t = t0; ok && t < t1; ++t) {
                    for (int kg = 0; kg < p.kchunks; kg += KPS, ++it) {
                        const int s = it % p.stages;
                        if (!mbar_wait(&ctl->empty[s], ((it / p.stages) & 1) ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        if (p.a.withhold_copy && it == 0) continue;  // test hook: never lands
                        mbar_arrive_expect_tx(&ctl->full[s], (uint32_t)(KPS * K3_STAGE_BYTES));
#pragma unroll
                        for (int j = 0; j < KPS; ++j)
                            tma_load_2d(ring + ((size_t)s * KPS + j) * K3_STAGE_BYTES, &tm_rows, &ctl->full[s],
                                        (kg + j) * KC, (int32_t)(t * K3_M));
                    }
                }
            }
            if (!ok) {
                atomicExch(p.a.err, ERR_TIMEOUT_TMA);
                *abort = 1;
            }
            // Every issued load must land before the block may exit.
            const uint32_t first = it > (uint32_t)p.stages ? it - p.stages : 0;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(&ctl->full[j % p.stages], (j / p.stages) & 1, nullptr);
            if (q_issued >= 0) mbar_wait(&ctl->qfull, q_issued & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            int uc = 0;
            bool ok = true;
            const uint32_t qbase = smem_u32(qsm);
            const uint32_t rbase = smem_u32(ring);
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
                int qt;
                int64_t t0, t1;
                unit_range(p, u, &qt, &t0, &t1);
                if (!mbar_wait(&ctl->qfull, uc & 1, abort)) { ok = false; break; }
                tc_fence_after();
                for (int64_t t = t0; ok && t < t1; ++t, ++tc) {
                    const int buf = tc & 1;
                    if (!mbar_wait(&ctl->tempty[buf], ((tc >> 1) & 1) ^ 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * K3_ACC_COLS);
                    for (int kg = 0; kg < p.kchunks; kg += KPS, ++it) {
                        const int s = it % p.stages;
                        if (!mbar_wait(&ctl->full[s], (it / p.stages) & 1, abort)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int j = 0; j < KPS; ++j) {
                            const int kc = kg + j;
                            const uint32_t a_addr = rbase + (uint32_t)((s * KPS + j) * K3_STAGE_BYTES);
                            const uint32_t b_addr = qbase + (uint32_t)(kc * q_chunk_bytes);
#pragma unroll
                            for (int kk = 0; kk < K3_ROW_BYTES / 32; ++kk) {  // 32 bytes of K per MMA
                                if constexpr (I8)
                                    umma_i8(d_tmem, umma_desc_kmajor_sw128(a_addr + kk * 32),
                                            umma_desc_kmajor_sw128(b_addr + kk * 32), p.idesc,
                                            (kc | kk) != 0 ? 1u : 0u);
                                else
                                    umma_bf16(d_tmem, umma_desc_kmajor_sw128(a_addr + kk * 32),
                                              umma_desc_kmajor_sw128(b_addr + kk * 32), p.idesc,
                                              (kc | kk) != 0 ? 1u : 0u);
                            }
                        }
                        umma_commit(&ctl->empty[s]);  // stage free once these MMAs finish
                    }
                    if (ok) umma_commit(&ctl->tfull[buf]);  // accumulator ready
                }
                if (ok) umma_commit(&ctl->qempty);  // query tile free after this unit
            }
            if (!ok) {
                atomicExch(p.a.err, ERR_TIMEOUT_MMA);
                *abort = 1;
            }
            // Wait for every MMA issued by this thread before TMEM is freed.
            umma_commit(&ctl->drain);
            mbar_wait(&ctl->drain, 0, nullptr);
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        // Warp w reads TMEM lanes 32*(w%4).. (its 32 corpus rows) and the
        // 32-column chunks half, half+2, half+4, half+6 of the query tile.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int row_in_tile = quarter * 32 + lane;
        const int nchunk32 = p.nq / 32;  // nq is a multiple of 32
        const PassArgs& a = p.a;
        // With no per-row norms the score scale c is the same for every row,
        // and the fast test compares the raw accumulator with th / c, lowered
        // by a relative 2^-20 so that fl(v * c) >= th implies v >= th_fast
        // (the exact test follows on the rare hits).
        const bool uniform_c = a.inv_norm == nullptr;
        float* th_fast = ctl->th_fast[ew];
        uint64_t* th_key = ctl->th_key[ew];
        float* q_us = ctl->q_us[ew];
        uint32_t tc = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            int qt;
            int64_t t0, t1;
            unit_range(p, u, &qt, &t0, &t1);
            const float* thf_unit = a.thf + (int64_t)qt * p.nq;
            const uint64_t* th_unit = a.theta + (int64_t)qt * p.nq;
            __syncwarp();
            for (int j = lane; j < K3_WARP_COLS; j += 32) {
                const int ch = half + 2 * (j >> 5);
                float t = INFINITY;
                th_key[j] = ch < nchunk32 ? __ldg(th_unit + ch * 32 + (j & 31)) : KEY_MAX;
                float us = 1.0f;
                if (ch < nchunk32) {
                    t = __ldg(thf_unit + ch * 32 + (j & 31));
                    if (I8) {
                        // score = fl(fl(acc * us) * c): the fast test compares
                        // fl(acc * c) with th / us, lowered like th / c below
                        const int q = qt * p.nq + ch * 32 + (j & 31);
                        us = q < a.b ? __ldg(a.qscale + q) : 1.0f;
                        if (t != INFINITY && t != -INFINITY) {
                            const float r = t / us;
                            t = r - fabsf(r) * 0x1p-20f - 1e-30f;
                        }
                    } else if (uniform_c && t != INFINITY && t != -INFINITY) {
                        const float r = t / a.inv_tau;
                        t = r - fabsf(r) * 0x1p-20f - 1e-30f;
                    }
                }
                th_fast[j] = t;
                q_us[j] = us;
            }
            __syncwarp();
            for (int64_t t = t0; t < t1; ++t, ++tc) {
                const int buf = tc & 1;
                // per-row data, fetched before waiting for the accumulator
                const int64_t j = t * K3_M + row_in_tile;
                const bool valid = j < a.n_rows;
                const int64_t id = j * a.stride;
                bool row_ok = valid;
                float c = a.inv_tau;
                int rset = 0;  // several result sets: this row's set
                if (valid) {
                    if (a.exclude) row_ok = !((a.exclude[id >> 5] >> (id & 31)) & 1u);
                    if (a.inv_norm) c = a.inv_norm[id] * a.inv_tau;
                    if (a.types) {
                        rset = a.set_of[a.types[id]];
                        if (rset < 0) row_ok = false;
                    }
                }
                if (!mbar_wait(&ctl->tfull[buf], (tc >> 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * K3_ACC_COLS);
                // this warp's chunks (up to 4 x 32 columns), two in flight per wait
                // (four would not fit the 168 registers a thread has here); a warp
                // whose half of the tile is empty releases the accumulator at once
                if (half >= nchunk32) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl->tempty[buf]);
                }
#pragma unroll
                for (int pair = 0; pair < 2; ++pair) {
                    const int cja = 2 * pair, cjb = 2 * pair + 1;
                    if (half + 2 * cja >= nchunk32) break;  // warp-uniform
                    const bool has_b = half + 2 * cjb < nchunk32;
                    Cols32 v[2];
                    tmem_ld_32cols(tbase + (uint32_t)((half + 2 * cja) * 32), v[0].x);
                    if (has_b) tmem_ld_32cols(tbase + (uint32_t)((half + 2 * cjb) * 32), v[1].x);
                    tmem_ld_wait();
                    if constexpr (I8) {  // int32 accumulators: exact in fp32 (|acc| < 2^24)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[h].x[i] = (float)__float_as_int(v[h].x[i]);
                    }
                    const bool last = pair == 1 || half + 2 * (cjb + 1) >= nchunk32;
                    if (last) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->tempty[buf]);  // values are in registers now
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int cj = cja + h;
                        if (h == 1 && !has_b) break;
                        const float4* t4 = reinterpret_cast<const float4*>(th_fast + cj * 32);
                        // four independent or-chains keep the compare latency short
                        bool h0 = false, h1 = false, h2 = false, h3 = false;
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 tf = t4[i4];
                            if (uniform_c) {
                                h0 |= v[h].x[4 * i4 + 0] >= tf.x;
                                h1 |= v[h].x[4 * i4 + 1] >= tf.y;
                                h2 |= v[h].x[4 * i4 + 2] >= tf.z;
                                h3 |= v[h].x[4 * i4 + 3] >= tf.w;
                            } else {
                                h0 |= v[h].x[4 * i4 + 0] * c >= tf.x;
                                h1 |= v[h].x[4 * i4 + 1] * c >= tf.y;
                                h2 |= v[h].x[4 * i4 + 2] * c >= tf.z;
                                h3 |= v[h].x[4 * i4 + 3] * c >= tf.w;
                            }
                        }
                        // Rare: only the lanes concerned find the passing columns
                        // and append those whose exact key beats the threshold key.
                        if ((h0 | h1 | h2 | h3) && row_ok) {
                            const int col0 = (half + 2 * cj) * 32;
                            const float cf = uniform_c ? 1.0f : c;
                            uint32_t m = 0;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                m |= (v[h].x[i] * cf >= th_fast[cj * 32 + i]) ? (1u << i) : 0u;
                            while (m) {
                                const int i = __ffs(m) - 1;
                                m &= m - 1;
                                const float acc = I8 ? select32(v[h], i) * q_us[cj * 32 + i] : select32(v[h], i);
                                const uint64_t key = make_key(acc * c, (uint32_t)id);
                                const int q = qt * p.nq + col0 + i;
                                if (a.types) {  // the row's set: its threshold and buffer
                                    if (q < a.b) {
                                        const int64_t v = (int64_t)rset * a.b + q;
                                        if (key > a.theta_v[v]) {
                                            const uint32_t slot = atomicAdd(a.count + v, 1u);
                                            if (slot < (uint32_t)a.cap) a.keys[v * a.cap + slot] = key;
                                        }
                                    }
                                } else if (key > th_key[cj * 32 + i]) {
                                    const uint32_t slot = atomicAdd(a.count + q, 1u);
                                    if (slot < (uint32_t)a.cap) a.keys[(int64_t)q * a.cap + slot] = key;
                                }
                            }
                        }
                    }
                }
            }
        }
        if (!ok) {
            atomicExch(a.err, ERR_TIMEOUT_EPI);
            *abort = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, K3_TMEM_COLS);
    }
}

}  // namespace

// K chunks per ring stage: two for rows of two chunks (one barrier handshake
// and one commit per tile: the 10^7 x 128, 32-query pass went from 0.56 to
// 0.53 ms), else one (rows of four chunks, 2*10^7 x 256 with 4096 queries,
// measured 8 % slower with two).
static int k3_kps(int kchunks, int fixed) {
    return (kchunks == 2 && (K3_SMEM_BUDGET - fixed) / (2 * K3_STAGE_BYTES) >= 3) ? 2 : 1;
}

int tensor_pass_smem_bytes(int d, int nq, int esize) {
    const int kchunks = (d * esize + K3_ROW_BYTES - 1) / K3_ROW_BYTES;
    const int q_bytes = kchunks * nq * 128;
    const int fixed = 1024 + q_bytes + (int)sizeof(K3Ctl);
    const int kps = k3_kps(kchunks, fixed);
    int stages = (K3_SMEM_BUDGET - fixed) / (kps * K3_STAGE_BYTES);
    if (stages > K3_MAX_STAGES) stages = K3_MAX_STAGES;
    if (stages < 2) return -1;
    return fixed + stages * kps * K3_STAGE_BYTES;
}

int tensor_pass_max_nq(int d, int esize) {
    for (int nq = K3_MAX_NQ; nq >= 32; nq -= 32)
        if (tensor_pass_smem_bytes(d, nq, esize) > 0 && tensor_pass_smem_bytes(d, nq, esize) <= K3_SMEM_BUDGET &&
            ((d * esize + K3_ROW_BYTES - 1) / K3_ROW_BYTES) * nq * 128 <= 128 * 1024)
            return nq;
    return 0;
}

cudaError_t launch_tensor_pass(const PassArgs& a, const CUtensorMap& tm_rows,
                               const CUtensorMap& tm_queries, int nq, cudaStream_t s,
                               int sm_count) {
    if (a.n_rows == 0 || a.b == 0) return cudaSuccess;
    K3Params p;
    p.a = a;
    p.nq = nq;
    p.q_tiles = (a.b + nq - 1) / nq;
    const bool i8 = a.dtype == TT_I8;
    const int esize = i8 ? 1 : 2;
    p.kchunks = (a.d * esize + K3_ROW_BYTES - 1) / K3_ROW_BYTES;
    const int smem = tensor_pass_smem_bytes(a.d, nq, esize);
    if (smem <= 0) return cudaErrorInvalidValue;
    const int fixed = 1024 + p.kchunks * nq * 128 + (int)sizeof(K3Ctl);
    p.kps = k3_kps(p.kchunks, fixed);
    p.stages = (smem - fixed) / (p.kps * K3_STAGE_BYTES);
    p.tiles = (a.n_rows + K3_M - 1) / K3_M;
    // Corpus chunks: make q_tiles * chunks a multiple of the SM count when
    // possible (every CTA gets the same number of units), with at least one
    // tile per chunk.
    int chunks = 0;
    for (int w = 1; w <= 8 && chunks == 0; ++w)
        if (((int64_t)sm_count * w) % p.q_tiles == 0) chunks = (int)((int64_t)sm_count * w / p.q_tiles);
    if (chunks == 0) chunks = (sm_count * 4 + p.q_tiles - 1) / p.q_tiles;
    if (chunks < 1) chunks = 1;
    if (chunks > p.tiles) chunks = (int)p.tiles;
    p.chunks = chunks;
    p.idesc = i8 ? umma_idesc_s8(K3_M, nq) : umma_idesc_bf16(K3_M, nq);
    const int n_units = p.q_tiles * p.chunks;
    const int grid = n_units < sm_count ? n_units : sm_count;
    auto kern = i8 ? (p.kps == 2 ? k3_tensor<true, 2> : k3_tensor<true, 1>)
                   : (p.kps == 2 ? k3_tensor<false, 2> : k3_tensor<false, 1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    note_launch_begin(TT_KIND_TENSOR, s);
    kern<<<grid, K3_THREADS, smem, s>>>(tm_rows, tm_queries, p);
    note_launch_end(TT_KIND_TENSOR, s);
    return cudaGetLastError();
}

}  // namespace tt
