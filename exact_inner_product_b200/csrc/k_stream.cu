// k_stream.cu - K2: small-batch streaming scorer on CUDA cores.
//
// For a handful of queries (b <= 8) scoring is bound by HBM bandwidth: the
// corpus must be read once and each row costs only b*d multiply-adds. One
// producer warp streams 32-row tiles of the corpus into a ring of shared-
// memory stages with TMA (128-byte swizzled boxes, so that a thread reading
// "its" row walks across all 32 banks); four consumer warps take one tile
// each, one thread per row, and form the dot products against the queries
// held in shared memory as fp32 (so fp32 queries keep full precision).
//
// Score and filter, per (query b, row j):
//   s = fl(dot * c_j), c_j = fl(inv_norm_j * inv_tau) (inv_norm_j = 1 when
//   the corpus is stored normalised); candidate kept iff it is not excluded
//   and key(s, j) > theta[b]. Kept keys are appended to the query's buffer;
//   the append is warp-aggregated (one atomicAdd per query per warp).
// (recsys_two_tower_model.py `forward`: scores = user . post_embeddings^T,
// masked candidates dropped; the top-k is taken from the kept keys by the
// select kernel.)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int K2_ROWS = 32;            // rows per tile (one per consumer lane)
constexpr int K2_CONSUMER_WARPS = 4;
constexpr int K2_THREADS = 32 * (K2_CONSUMER_WARPS + 1);
constexpr int K2_MAX_QB = 8;

struct K2Smem {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t theta[K2_MAX_QB];
    int abort;
};

__device__ __forceinline__ void unpack16(const uint4& c, float* x, float) {
    x[0] = __uint_as_float(c.x);
    x[1] = __uint_as_float(c.y);
    x[2] = __uint_as_float(c.z);
    x[3] = __uint_as_float(c.w);
}
__device__ __forceinline__ void unpack16(const uint4& c, float* x, __nv_bfloat16) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// T: corpus element type. QB: queries per block. SW: rows are >= 128 bytes
// and staged as 128-byte swizzled boxes (else one unswizzled box per row).
template <typename T, int QB, bool SW>
__global__ void __launch_bounds__(K2_THREADS)
    k2_stream(const __grid_constant__ CUtensorMap tm_rows, const PassArgs a, int ntiles,
              int nbox, int stages, int row_pitch, int d_pad) {
    constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = K2_ROWS * row_pitch;  // multiple of 1024 when SW
    uint8_t* ring = smem;
    float* qs = reinterpret_cast<float*>(ring + (size_t)stages * stage_bytes);  // [QB][d_pad]
    K2Smem* ctl = reinterpret_cast<K2Smem*>(qs + QB * d_pad);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.y * QB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        ctl->abort = 0;
        fence_barrier_init();
    }
    // Stage this block's queries as fp32, zero-padded to d_pad.
    for (int i = threadIdx.x; i < QB * d_pad; i += blockDim.x) {
        const int qb = i / d_pad, e = i % d_pad;
        float v = 0.f;
        if (q0 + qb < a.b && e < a.d) {
            const int64_t off = (int64_t)(q0 + qb) * a.d + e;
            v = a.q_dtype == TT_F32 ? static_cast<const float*>(a.queries)[off]
                                    : __bfloat162float(static_cast<const __nv_bfloat16*>(a.queries)[off]);
        }
        qs[i] = v;
    }
    if (threadIdx.x < QB) ctl->theta[threadIdx.x] = (q0 + threadIdx.x < a.b) ? a.theta[q0 + threadIdx.x] : KEY_MAX;
    __syncthreads();

    volatile int* abort = &ctl->abort;
    const int tiles_here = ntiles > (int)blockIdx.x
                               ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                               : 0;

    if (warp == K2_CONSUMER_WARPS) {
        // ---------------- producer ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_rows);
            int i = 0;
            for (; i < tiles_here; ++i) {
                const int s = i % stages;
                if (!mbar_wait(&ctl->empty[s], ((i / stages) & 1) ^ 1, abort)) {
                    atomicExch(a.err, ERR_TIMEOUT_STREAM);
                    *abort = 1;
                    break;
                }
                const int t = blockIdx.x + i * gridDim.x;
                mbar_arrive_expect_tx(&ctl->full[s], stage_bytes);
                uint8_t* dst = ring + (size_t)s * stage_bytes;
                if (SW) {
                    for (int bx = 0; bx < nbox; ++bx)
                        tma_load_2d(dst + bx * (K2_ROWS * 128), &tm_rows, &ctl->full[s],
                                    bx * (128 / (int)sizeof(T)), t * K2_ROWS);
                } else {
                    tma_load_2d(dst, &tm_rows, &ctl->full[s], 0, t * K2_ROWS);
                }
            }
            // Every load issued must land before the block may exit.
            for (int j = (i > stages ? i - stages : 0); j < i; ++j)
                mbar_wait(&ctl->full[j % stages], (j / stages) & 1, nullptr);
        }
    } else {
        // ---------------- consumers: one tile per warp, one row per lane ----------------
        for (int i = warp; i < tiles_here; i += K2_CONSUMER_WARPS) {
            const int s = i % stages;
            if (!mbar_wait(&ctl->full[s], (i / stages) & 1, abort)) {
                atomicExch(a.err, ERR_TIMEOUT_STREAM);
                *abort = 1;
                break;
            }
            const uint8_t* st = ring + (size_t)s * stage_bytes;
            float acc[QB];
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) acc[qb] = 0.f;
            const int nchunks = d_pad / E;
#pragma unroll 4
            for (int c = 0; c < nchunks; ++c) {
                const uint8_t* p;
                if (SW) {
                    const int bx = c >> 3, cc = c & 7;
                    p = st + bx * (K2_ROWS * 128) + lane * 128 + ((cc ^ (lane & 7)) << 4);
                } else {
                    p = st + lane * row_pitch + (c << 4);
                }
                const uint4 raw = *reinterpret_cast<const uint4*>(p);
                float x[E];
                unpack16(raw, x, T());
#pragma unroll
                for (int qb = 0; qb < QB; ++qb) {
                    const float4* qv = reinterpret_cast<const float4*>(qs + qb * d_pad + c * E);
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
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->empty[s]);

            // ---------- filter and append ----------
            const int t = blockIdx.x + i * gridDim.x;
            const int64_t j = (int64_t)t * K2_ROWS + lane;
            const bool valid = j < a.n_rows;
            const int64_t id = j * a.stride;
            bool excluded = false;
            float c = a.inv_tau;
            if (valid) {
                if (a.exclude) excluded = (a.exclude[id >> 5] >> (id & 31)) & 1u;
                if (a.inv_norm) c = a.inv_norm[id] * a.inv_tau;
            }
#pragma unroll
            for (int qb = 0; qb < QB; ++qb) {
                const float sc = acc[qb] * c;
                const uint64_t key = make_key(sc, (uint32_t)id);
                const bool keep = valid && !excluded && key > ctl->theta[qb];
                const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, keep);
                if (ballot) {
                    const int q = q0 + qb;
                    uint32_t base = 0;
                    const int leader = __ffs(ballot) - 1;
                    if (lane == leader) base = atomicAdd(a.count + q, (uint32_t)__popc(ballot));
                    base = __shfl_sync(0xFFFFFFFFu, base, leader);
                    if (keep) {
                        const uint32_t slot = base + __popc(ballot & lanemask_lt());
                        if (slot < (uint32_t)a.cap) a.keys[(int64_t)q * a.cap + slot] = key;
                    }
                }
            }
        }
    }
    __syncthreads();
}

template <typename T, int QB>
cudaError_t launch_qb(const PassArgs& a, const CUtensorMap& tm, int ntiles, int nbox, int stages,
                      int row_pitch, int d_pad, bool sw, int grid_x, int grid_y, size_t smem,
                      cudaStream_t s) {
    if (sw) {
        auto kern = k2_stream<T, QB, true>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<dim3(grid_x, grid_y), K2_THREADS, smem, s>>>(tm, a, ntiles, nbox, stages, row_pitch, d_pad);
    } else {
        auto kern = k2_stream<T, QB, false>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<dim3(grid_x, grid_y), K2_THREADS, smem, s>>>(tm, a, ntiles, nbox, stages, row_pitch, d_pad);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const PassArgs& a, const CUtensorMap& tm, int qb, int ntiles, int nbox,
                     int stages, int row_pitch, int d_pad, bool sw, int gx, int gy, size_t smem,
                     cudaStream_t s) {
    switch (qb) {
        case 1: return launch_qb<T, 1>(a, tm, ntiles, nbox, stages, row_pitch, d_pad, sw, gx, gy, smem, s);
        case 2: return launch_qb<T, 2>(a, tm, ntiles, nbox, stages, row_pitch, d_pad, sw, gx, gy, smem, s);
        case 4: return launch_qb<T, 4>(a, tm, ntiles, nbox, stages, row_pitch, d_pad, sw, gx, gy, smem, s);
        default: return launch_qb<T, 8>(a, tm, ntiles, nbox, stages, row_pitch, d_pad, sw, gx, gy, smem, s);
    }
}

}  // namespace

cudaError_t launch_stream_pass(const PassArgs& a, cudaStream_t s, int sm_count) {
    if (a.n_rows == 0 || a.b == 0) return cudaSuccess;
    CUtensorMap tm;
    int nbox = 0, row_pitch = 0;
    bool sw = false;
    if (!stream_pass_tensor_map(a, &tm, &nbox, &row_pitch, &sw)) return cudaErrorInvalidValue;
    const int elem = a.dtype == TT_F32 ? 4 : 2;
    const int d_pad = row_pitch / elem;
    const int stage_bytes = K2_ROWS * row_pitch;
    int stages = (128 * 1024) / stage_bytes;
    stages = stages >= 16 ? 16 : (stages >= 8 ? 8 : 4);
    const int qb = a.b >= 8 ? 8 : (a.b >= 4 ? (a.b == 4 ? 4 : 8) : (a.b == 1 ? 1 : (a.b == 2 ? 2 : 4)));
    const size_t smem = 1024 + (size_t)stages * stage_bytes + (size_t)qb * d_pad * 4 + sizeof(K2Smem);
    const int64_t ntiles64 = (a.n_rows + K2_ROWS - 1) / K2_ROWS;
    const int ntiles = (int)ntiles64;
    const int blocks_per_sm = (int)((227 * 1024) / smem) > 0 ? (int)((227 * 1024) / smem) : 1;
    const int gy = (a.b + qb - 1) / qb;
    int64_t gx = (int64_t)sm_count * (blocks_per_sm > 4 ? 4 : blocks_per_sm);
    gx = (gx + gy - 1) / gy;
    if (gx > ntiles) gx = ntiles;
    if (gx < 1) gx = 1;
    note_launch_begin(TT_KIND_STREAM, s);
    cudaError_t e = a.dtype == TT_F32
                        ? launch_t<float>(a, tm, qb, ntiles, nbox, stages, row_pitch, d_pad, sw, (int)gx, gy, smem, s)
                        : launch_t<__nv_bfloat16>(a, tm, qb, ntiles, nbox, stages, row_pitch, d_pad, sw, (int)gx, gy, smem, s);
    note_launch_end(TT_KIND_STREAM, s);
    return e;
}

}  // namespace tt
