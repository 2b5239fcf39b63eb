// k_stream.cu - K2: small-batch streaming scorer on CUDA cores.
//
// For a handful of queries (b <= 8), or an fp32 corpus, scoring is bound by
// HBM bandwidth: the corpus is read once and each row costs only b*d
// multiply-adds. One thread scores one row at a time. It reads the row with
// 256-bit loads (a warp's load instruction fetches 32 whole 32-byte sectors,
// one per row), up to eight of them in flight before the first is used, and
// forms the dot products against the queries, which every block stages in
// shared memory as fp32 (an fp32 query keeps full precision; all lanes read
// the same query word, a broadcast). Because each lane owns a whole row, the
// filter below runs with all 32 lanes busy and needs no reduction.
//
// Score and filter, per (query b, row j):
//   s = fl(dot * c_j), c_j = fl(inv_norm_j * inv_tau) (inv_norm_j = 1 when
//   the corpus is stored normalised); candidate kept iff it is not excluded
//   and key(s, j) > theta[b].
// int8 rows (k2_stream_i8; recsys_two_tower_model.py `compute_top_k_int8`):
//   the queries are int8 codes with scales us_b, staged as packed words; dot
//   is the exact int32 sum of code products (dp4a), s = fl(fl(fl(dot) * us_b)
//   * c_j) with c_j = fl(scale_j * inv_tau). Kept keys are appended to the query's buffer;
//   the append is warp-aggregated (one atomicAdd per query per warp).
// Several result sets by candidate type: the first test uses the query's
//   loosest set threshold; a key that passes goes to its row's set if it
//   beats that set's threshold.
// (recsys_two_tower_model.py `forward`: scores = user . post_embeddings^T,
// masked candidates dropped; the top-k is taken from the kept keys by the
// select kernel.)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int K2_THREADS = 256;
constexpr int K2_BATCH = 8;  // 32-byte loads in flight per thread
constexpr int K2_MAX_QB = 8;
constexpr int K2_DEFER = 4;  // rows per thread scored before the threshold is known

struct Raw32 {
    uint32_t w[8];
};

// 32 bytes of a row, read once. V8: the address is 32-byte aligned (one
// 256-bit load), else two 128-bit loads.
template <bool V8>
__device__ __forceinline__ Raw32 ld32(const uint8_t* p) {
    Raw32 r;
    if (V8) {
        asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                       "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
                     : "l"(p));
    } else {
        const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p));
        const uint4 b = __ldcs(reinterpret_cast<const uint4*>(p + 16));
        r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
        r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
    }
    return r;
}

// Elements of a 32-byte piece as fp32.
__device__ __forceinline__ void unpack32(const Raw32& r, float* x, float) {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = __uint_as_float(r.w[i]);
}
__device__ __forceinline__ void unpack32(const Raw32& r, float* x, __nv_bfloat16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(r.w[i] << 16);
        x[2 * i + 1] = __uint_as_float(r.w[i] & 0xFFFF0000u);
    }
}

// Several result sets: a key that beat the query's loosest set threshold is
// kept if it beats the threshold of its row's set, in that set's buffer.
__device__ __forceinline__ void append_set(const PassArgs& a, int q, int rset, bool keep, uint64_t key) {
    if (!keep) return;
    const int64_t v = (int64_t)rset * a.b + q;
    if (key > a.theta_v[v]) {
        const uint32_t slot = atomicAdd(a.count + v, 1u);
        if (slot < (uint32_t)a.cap) a.keys[v * a.cap + slot] = key;
    }
}

// Kept keys of one warp appended to query q's buffer (warp-aggregated).
__device__ __forceinline__ void append_warp(const PassArgs& a, int q, bool keep, uint64_t key, int lane) {
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, keep);
    if (ballot) {
        const int leader = __ffs(ballot) - 1;
        uint32_t slot0 = 0;
        if (lane == leader) slot0 = atomicAdd(a.count + q, (uint32_t)__popc(ballot));
        slot0 = __shfl_sync(0xFFFFFFFFu, slot0, leader);
        if (keep) {
            const uint32_t slot = slot0 + __popc(ballot & lanemask_lt());
            if (slot < (uint32_t)a.cap) a.keys[(int64_t)q * a.cap + slot] = key;
        }
    }
}

// T: corpus element type. QB: queries per block (blockIdx.y selects the
// group). V8: rows start on 32-byte boundaries. PF: the whole row fits one
// batch of loads, and the next row's loads are issued before the current
// row is scored (used when every thread streams many rows: on 10^7 rows of
// 256 bytes it raised the pass from 5.5 to 6.1 TB/s; with only three or four
// rows per thread, as on 10^6 rows, it was slower).
// DEFER > 0: the pass follows the one-sample estimate of its threshold. Each
// thread scores its first DEFER rows before it waits for that kernel, keeps
// their keys in registers and filters them once the threshold is known, so
// the first blocks stream rows while the estimate runs. Reading the rows and
// the queries before the wait is safe: no kernel that writes them signals its
// dependents early, so the search's first kernel, and with it every later
// one, starts only after those writes completed.
template <typename T, int QB, bool V8, bool PF, int DEFER>
__global__ void __launch_bounds__(K2_THREADS)
    k2_stream(const PassArgs a) {
    constexpr int E = 32 / (int)sizeof(T);  // elements per 32-byte piece
    extern __shared__ __align__(16) float qs[];  // [QB][d]
    pdl_trigger();
    if (DEFER == 0) pdl_wait();  // queries, thresholds and counters come from earlier kernels
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.y * QB;
    const int d = a.d;
    const int pieces = d / E;  // d % 16 == 0: a whole number of pieces
    for (int i = threadIdx.x; i < QB * d; i += blockDim.x) {
        const int qb = i / d, e = i % d;
        const int q = q0 + qb;
        float v = 0.f;
        if (q < a.b) {
            const int64_t off = (int64_t)q * d + e;
            v = a.q_dtype == TT_F32 ? static_cast<const float*>(a.queries)[off]
                                    : __bfloat162float(static_cast<const __nv_bfloat16*>(a.queries)[off]);
        }
        qs[i] = v;
    }
    __syncthreads();

    const int64_t pitch = (int64_t)a.stride * d * (int)sizeof(T);
    const uint8_t* base = static_cast<const uint8_t*>(a.rows);
    const int64_t n_threads = (int64_t)gridDim.x * blockDim.x;
    int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint64_t th[QB];
    if constexpr (DEFER > 0) {
        uint64_t kb[DEFER][QB];  // keys of the first DEFER rows (KEY_MIN: no row, or excluded)
#pragma unroll
        for (int i = 0; i < DEFER; ++i, r += n_threads) {
            const bool valid = r < a.n_rows;
            const uint8_t* row = base + (valid ? r : 0) * pitch;
            float acc[QB];
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) acc[qb] = 0.f;
            for (int p0 = 0; p0 < pieces; p0 += K2_BATCH) {
                Raw32 raw[K2_BATCH];
#pragma unroll
                for (int j = 0; j < K2_BATCH; ++j)
                    if (p0 + j < pieces && valid) raw[j] = ld32<V8>(row + (int64_t)(p0 + j) * 32);
#pragma unroll
                for (int j = 0; j < K2_BATCH; ++j) {
                    if (p0 + j >= pieces) break;
                    float x[E];
                    unpack32(raw[j], x, T());
                    const int e0 = (p0 + j) * E;
#pragma unroll
                    for (int qb = 0; qb < QB; ++qb) {
                        const float4* qv = reinterpret_cast<const float4*>(qs + qb * d + e0);
#pragma unroll
                        for (int v4 = 0; v4 < E / 4; ++v4) {
                            const float4 q = qv[v4];
                            acc[qb] = fmaf(x[4 * v4 + 0], q.x, acc[qb]);
                            acc[qb] = fmaf(x[4 * v4 + 1], q.y, acc[qb]);
                            acc[qb] = fmaf(x[4 * v4 + 2], q.z, acc[qb]);
                            acc[qb] = fmaf(x[4 * v4 + 3], q.w, acc[qb]);
                        }
                    }
                }
            }
            const int64_t id = r * a.stride;
            bool row_ok = valid;
            float c = a.inv_tau;
            if (valid) {
                if (a.exclude) row_ok = !((a.exclude[id >> 5] >> (id & 31)) & 1u);
                if (a.inv_norm) c = a.inv_norm[id] * a.inv_tau;
            }
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) kb[i][qb] = row_ok ? make_key(acc[qb] * c, (uint32_t)id) : KEY_MIN;
        }
        pdl_wait();  // this pass's thresholds
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) th[qb] = (q0 + qb < a.b) ? a.theta[q0 + qb] : KEY_MAX;
#pragma unroll
        for (int i = 0; i < DEFER; ++i)
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) append_warp(a, q0 + qb, kb[i][qb] > th[qb], kb[i][qb], lane);
    } else {
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) th[qb] = (q0 + qb < a.b) ? a.theta[q0 + qb] : KEY_MAX;
    }
    // whole warps step together so the ballots below see every lane
    Raw32 nxt[PF ? K2_BATCH : 1];
    if (PF) {
        if (r < a.n_rows)
#pragma unroll
            for (int j = 0; j < K2_BATCH; ++j)
                if (j < pieces) nxt[j] = ld32<V8>(base + r * pitch + (int64_t)j * 32);
    }
    for (; r - lane < a.n_rows; r += n_threads) {
        const bool valid = r < a.n_rows;
        const uint8_t* row = base + (valid ? r : 0) * pitch;
        float acc[QB];
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) acc[qb] = 0.f;
        for (int p0 = 0; p0 < pieces; p0 += K2_BATCH) {
            Raw32 raw[K2_BATCH];
            if (PF) {  // this row was loaded one step ahead; load the next
#pragma unroll
                for (int j = 0; j < K2_BATCH; ++j) raw[j] = nxt[j];
                if (r + n_threads < a.n_rows)
#pragma unroll
                    for (int j = 0; j < K2_BATCH; ++j)
                        if (j < pieces) nxt[j] = ld32<V8>(base + (r + n_threads) * pitch + (int64_t)j * 32);
            } else {
#pragma unroll
                for (int j = 0; j < K2_BATCH; ++j)
                    if (p0 + j < pieces && valid) raw[j] = ld32<V8>(row + (int64_t)(p0 + j) * 32);
            }
#pragma unroll
            for (int j = 0; j < K2_BATCH; ++j) {
                if (p0 + j >= pieces) break;
                float x[E];
                unpack32(raw[j], x, T());
                const int e0 = (p0 + j) * E;
#pragma unroll
                for (int qb = 0; qb < QB; ++qb) {
                    const float4* qv = reinterpret_cast<const float4*>(qs + qb * d + e0);
#pragma unroll
                    for (int v4 = 0; v4 < E / 4; ++v4) {
                        const float4 q = qv[v4];
                        acc[qb] = fmaf(x[4 * v4 + 0], q.x, acc[qb]);
                        acc[qb] = fmaf(x[4 * v4 + 1], q.y, acc[qb]);
                        acc[qb] = fmaf(x[4 * v4 + 2], q.z, acc[qb]);
                        acc[qb] = fmaf(x[4 * v4 + 3], q.w, acc[qb]);
                    }
                }
            }
        }
        // filter and append
        const int64_t id = r * a.stride;
        bool row_ok = valid;
        float c = a.inv_tau;
        int rset = 0;
        if (valid) {
            if (a.exclude) row_ok = !((a.exclude[id >> 5] >> (id & 31)) & 1u);
            if (a.inv_norm) c = a.inv_norm[id] * a.inv_tau;
            if (a.types) {
                rset = a.set_of[a.types[id]];
                if (rset < 0) row_ok = false;
            }
        }
        if (a.types) {  // this row's set: its own threshold and buffer
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) {
                const uint64_t key = make_key(acc[qb] * c, (uint32_t)id);
                append_set(a, q0 + qb, rset, row_ok && key > th[qb], key);
            }
            continue;
        }
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) {
            const uint64_t key = make_key(acc[qb] * c, (uint32_t)id);
            append_warp(a, q0 + qb, row_ok && key > th[qb], key, lane);
        }
    }
}

// int8 rows: one thread per row, 32 codes per 32-byte piece, dp4a against
// the staged query code words. d % 32 == 0; four pieces (128 codes) in
// flight per thread.
constexpr int K2_BATCH_I8 = 4;

template <int QB, bool V8, int DEFER>
__global__ void __launch_bounds__(K2_THREADS)
    k2_stream_i8(const PassArgs a) {
    extern __shared__ __align__(16) int qw[];  // [QB][d / 4] packed codes
    pdl_trigger();
    // DEFER > 0: as in k2_stream, the first DEFER rows of each thread are
    // scored before the wait (the query codes and scales are written by the
    // query coding, which completes before the search's next kernel starts)
    if (DEFER == 0) pdl_wait();  // query codes, thresholds and counters come from earlier kernels
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.y * QB;
    const int d = a.d;
    const int dw = d / 4;
    const int pieces = d / 32;
    for (int i = threadIdx.x; i < QB * dw; i += blockDim.x) {
        const int qb = i / dw, w = i % dw;
        const int q = q0 + qb;
        qw[i] = q < a.b ? reinterpret_cast<const int*>(a.queries)[(int64_t)q * dw + w] : 0;
    }
    float us[QB];
#pragma unroll
    for (int qb = 0; qb < QB; ++qb) us[qb] = (q0 + qb < a.b) ? a.qscale[q0 + qb] : 1.0f;
    __syncthreads();

    const int64_t pitch = (int64_t)a.stride * d;
    const uint8_t* base = static_cast<const uint8_t*>(a.rows);
    const int64_t n_threads = (int64_t)gridDim.x * blockDim.x;
    // the int32 dot products of row r with this block's query codes
    auto dots = [&](int64_t r, bool valid, int* acc) {
        const uint8_t* row = base + (valid ? r : 0) * pitch;
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) acc[qb] = 0;
        for (int p0 = 0; p0 < pieces; p0 += K2_BATCH_I8) {
            Raw32 raw[K2_BATCH_I8];
#pragma unroll
            for (int j = 0; j < K2_BATCH_I8; ++j)
                if (p0 + j < pieces && valid) raw[j] = ld32<V8>(row + (int64_t)(p0 + j) * 32);
#pragma unroll
            for (int j = 0; j < K2_BATCH_I8; ++j) {
                if (p0 + j >= pieces) break;
                const int w0 = (p0 + j) * 8;
#pragma unroll
                for (int qb = 0; qb < QB; ++qb) {
                    const int4* qv = reinterpret_cast<const int4*>(qw + qb * dw + w0);
                    const int4 qa = qv[0], qc = qv[1];
                    acc[qb] = __dp4a((int)raw[j].w[0], qa.x, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[1], qa.y, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[2], qa.z, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[3], qa.w, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[4], qc.x, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[5], qc.y, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[6], qc.z, acc[qb]);
                    acc[qb] = __dp4a((int)raw[j].w[7], qc.w, acc[qb]);
                }
            }
        }
    };
    int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint64_t th[QB];
    if constexpr (DEFER > 0) {
        uint64_t kb[DEFER][QB];  // keys of the first DEFER rows (KEY_MIN: no row, or excluded)
#pragma unroll
        for (int i = 0; i < DEFER; ++i, r += n_threads) {
            const bool valid = r < a.n_rows;
            int acc[QB];
            dots(r, valid, acc);
            const int64_t id = r * a.stride;
            bool row_ok = valid;
            float c = a.inv_tau;
            if (valid) {
                if (a.exclude) row_ok = !((a.exclude[id >> 5] >> (id & 31)) & 1u);
                c = a.inv_norm[id] * a.inv_tau;
            }
#pragma unroll
            for (int qb = 0; qb < QB; ++qb)
                kb[i][qb] = row_ok ? make_key((float)acc[qb] * us[qb] * c, (uint32_t)id) : KEY_MIN;
        }
        pdl_wait();  // this pass's thresholds
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) th[qb] = (q0 + qb < a.b) ? a.theta[q0 + qb] : KEY_MAX;
#pragma unroll
        for (int i = 0; i < DEFER; ++i)
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) append_warp(a, q0 + qb, kb[i][qb] > th[qb], kb[i][qb], lane);
    } else {
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) th[qb] = (q0 + qb < a.b) ? a.theta[q0 + qb] : KEY_MAX;
    }

    for (; r - lane < a.n_rows; r += n_threads) {
        const bool valid = r < a.n_rows;
        int acc[QB];
        dots(r, valid, acc);
        const int64_t id = r * a.stride;
        bool row_ok = valid;
        float c = a.inv_tau;
        int rset = 0;
        if (valid) {
            if (a.exclude) row_ok = !((a.exclude[id >> 5] >> (id & 31)) & 1u);
            c = a.inv_norm[id] * a.inv_tau;
            if (a.types) {
                rset = a.set_of[a.types[id]];
                if (rset < 0) row_ok = false;
            }
        }
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) {
            // |acc| < 2^24 (127 * 127 * 512), so fl(acc) is exact
            const uint64_t key = make_key((float)acc[qb] * us[qb] * c, (uint32_t)id);
            if (a.types)
                append_set(a, q0 + qb, rset, row_ok && key > th[qb], key);
            else
                append_warp(a, q0 + qb, row_ok && key > th[qb], key, lane);
        }
    }
}

// Grid of a streaming pass: one block per 256 rows, at most 8 blocks of 256 threads per SM
// (blocks loop over their rows). Measured on the 10^6-row pass: a grid of
// exactly the resident blocks (each looping ~13 times) took 53 us against 47
// us for this one, which runs in about four waves of resident blocks.
template <typename K>
dim3 stream_grid(K, const PassArgs& a, int gy, size_t, int sm_count) {
    int64_t gx = (a.n_rows + K2_THREADS - 1) / K2_THREADS;
    int64_t max_gx = ((int64_t)sm_count * (2048 / K2_THREADS) + gy - 1) / gy;
    if (gx > max_gx) gx = max_gx;
    if (gx < 1) gx = 1;
    return dim3((unsigned)gx, (unsigned)gy);
}

template <typename T, int QB, bool V8>
cudaError_t launch_qbv(const PassArgs& a, int gy, size_t smem, cudaStream_t s, int sms) {
    const dim3 grid = stream_grid(k2_stream<T, QB, V8, false, 0>, a, gy, smem, sms);
    constexpr int E = 32 / (int)sizeof(T);
    const bool one_batch = a.d / E <= K2_BATCH;
    const int64_t rows_per_thread = a.n_rows / ((int64_t)grid.x * K2_THREADS);
    if (one_batch && rows_per_thread >= 8)
        return launch_pdl(k2_stream<T, QB, V8, true, 0>, grid, dim3(K2_THREADS), smem, s, a);
    // after the one-sample estimate: the first rows are scored while it runs
    if constexpr (QB <= 2) {
        if (a.defer && a.types == nullptr)
            return launch_pdl(k2_stream<T, QB, V8, false, K2_DEFER>, grid, dim3(K2_THREADS), smem, s, a);
    }
    return launch_pdl(k2_stream<T, QB, V8, false, 0>, grid, dim3(K2_THREADS), smem, s, a);
}

template <typename T, int QB>
cudaError_t launch_qb(const PassArgs& a, int gy, size_t smem, bool v8, cudaStream_t s, int sms) {
    return v8 ? launch_qbv<T, QB, true>(a, gy, smem, s, sms) : launch_qbv<T, QB, false>(a, gy, smem, s, sms);
}

template <int QB, bool V8>
cudaError_t launch_i8_qbv(const PassArgs& a, int gy, size_t smem, cudaStream_t s, int sms) {
    const dim3 grid = stream_grid(k2_stream_i8<QB, V8, 0>, a, gy, smem, sms);
    // after the one-sample estimate: the first rows are scored while it runs
    if constexpr (QB <= 2) {
        if (a.defer && a.types == nullptr)
            return launch_pdl(k2_stream_i8<QB, V8, K2_DEFER>, grid, dim3(K2_THREADS), smem, s, a);
    }
    return launch_pdl(k2_stream_i8<QB, V8, 0>, grid, dim3(K2_THREADS), smem, s, a);
}

template <int QB>
cudaError_t launch_i8_qb(const PassArgs& a, int gy, size_t smem, bool v8, cudaStream_t s, int sms) {
    return v8 ? launch_i8_qbv<QB, true>(a, gy, smem, s, sms) : launch_i8_qbv<QB, false>(a, gy, smem, s, sms);
}

cudaError_t launch_i8(const PassArgs& a, int qb, int gy, size_t smem, bool v8, cudaStream_t s, int sms) {
    switch (qb) {
        case 1: return launch_i8_qb<1>(a, gy, smem, v8, s, sms);
        case 2: return launch_i8_qb<2>(a, gy, smem, v8, s, sms);
        case 4: return launch_i8_qb<4>(a, gy, smem, v8, s, sms);
        default: return launch_i8_qb<8>(a, gy, smem, v8, s, sms);
    }
}

template <typename T>
cudaError_t launch_t(const PassArgs& a, int qb, int gy, size_t smem, bool v8, cudaStream_t s, int sms) {
    switch (qb) {
        case 1: return launch_qb<T, 1>(a, gy, smem, v8, s, sms);
        case 2: return launch_qb<T, 2>(a, gy, smem, v8, s, sms);
        case 4: return launch_qb<T, 4>(a, gy, smem, v8, s, sms);
        default: return launch_qb<T, 8>(a, gy, smem, v8, s, sms);
    }
}

}  // namespace

cudaError_t launch_stream_pass(const PassArgs& a, cudaStream_t s, int sm_count) {
    if (a.n_rows == 0 || a.b == 0) return cudaSuccess;
    const int qb = a.b >= 8 ? K2_MAX_QB : (a.b >= 4 ? (a.b == 4 ? 4 : 8) : (a.b == 1 ? 1 : (a.b == 2 ? 2 : 4)));
    const int gy = (a.b + qb - 1) / qb;
    const size_t smem = (size_t)qb * a.d * sizeof(float);
    const bool v8 = (reinterpret_cast<uintptr_t>(a.rows) % 32) == 0;
    note_launch_begin(TT_KIND_STREAM, s);
    cudaError_t e = a.dtype == TT_F32    ? launch_t<float>(a, qb, gy, smem, v8, s, sm_count)
                    : a.dtype == TT_I8 ? launch_i8(a, qb, gy, smem, v8, s, sm_count)
                                       : launch_t<__nv_bfloat16>(a, qb, gy, smem, v8, s, sm_count);
    note_launch_end(TT_KIND_STREAM, s);
    return e;
}

}  // namespace tt
