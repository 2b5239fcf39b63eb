// k_softmax.cu - K5: in-batch sampled softmax (the training loss) on the
// 5th-generation tensor cores, without writing the b x nc logit matrix.
//
// Row i of the batch is a user u_i whose positive is candidate i; every
// other candidate column is a negative ("Two-Tower Retrieval at Industrial
// Scale", section 3, In-batch sampled softmax: logits = U V^T / tau, labels
// = arange(B), cross-entropy). Columns j >= b are negatives shared by every
// row (the global negatives of x-algorithm recsys_two_tower_model.py
// `compute_retrieval_loss`). The corrected logit subtracts log q_j on every
// column, the positive included (same article, section 4, The LogQ
// Correction, `corrected_in_batch_loss`); a column j != i holding the same
// item as row i (an accidental hit) and an invalid column are left out of
// row i's denominator. Outputs: lse_i = log sum_j exp(l_ij), loss_i =
// lse_i - l_ii for valid rows (0 otherwise), and the mean loss over valid
// rows (`compute_retrieval_loss`: log_denominator - numerator_logits,
// averaged).
//
// Kernels, in launch order:
//   k5_table_clear  (with item ids) empty the open-addressing table
//   k5_columns      per column: bias nb_j = -log q_j * log2(e) (-inf for an
//                   invalid column) and item group g_j (the table slot of its
//                   id, so equal ids <=> equal groups); zero the error word
//   k5_softmax      tcgen05 MMAs of 128 users x 256 candidates into TMEM;
//                   the epilogue turns each accumulator row into running
//                   (max, sum of 2^(x - max)) pairs, x = acc * log2(e)/tau + nb_j,
//                   so the exponentials never leave registers
//   k5_merge        per row: combine the partial pairs (and, with item ids,
//                   the diagonal term the group test left out), lse, loss,
//                   and the mean over valid rows in a fixed order
//
// The epilogue runs in base-2 units so that each term is one ex2.approx
// (MUFU) instruction; that unit, 16 results per clock per SM, bounds the
// kernel at d <= 128, not the tensor cores.
//
// Every wait is bounded; on expiry the kernel records an error code, the
// merge writes NaN to every output, and the host check reports a timeout.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int K5_M = 128;                    // users per tile (TMEM lanes)
constexpr int K5_N = 256;                    // candidates per tile (TMEM columns)
constexpr int K5_USER_CHUNK = K5_M * 128;    // one 128-byte K chunk of the user tile
constexpr int K5_STAGE_BYTES = K5_N * 128;   // one 128-byte K chunk of a candidate tile
constexpr int K5_MAX_STAGES = 8;
constexpr int K5_EPI_WARPS = 8;
constexpr int K5_THREADS = 32 * (2 + K5_EPI_WARPS);
constexpr int K5_TMEM_COLS = 512;
constexpr int K5_ACC_COLS = 256;
constexpr int K5_SMEM_BUDGET = 227 * 1024;
constexpr int K5_HALF = K5_N / 2;            // columns of one epilogue warp
constexpr float K5_MAX_FLOOR = -1e30f;       // running max before any column (base-2 units)
constexpr float K5_LAG = 8.0f;               // the running max may trail the true one by 8
constexpr float K5_LOG2E = 1.4426950408889634f;
constexpr float K5_LN2 = 0.6931471805599453f;
constexpr unsigned long long K5_EMPTY = 0x8000000000000000ull;  // free table slot
constexpr int K5_MERGE_THREADS = 256;

struct alignas(8) ColInfo {
    float nb;  // -log q_j * log2(e), or -inf when the column is invalid or past nc
    int g;     // item group
};

struct K5Ctl {
    uint64_t full[K5_MAX_STAGES];
    uint64_t empty[K5_MAX_STAGES];
    uint64_t ufull, uempty;
    uint64_t tfull[2], tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    // per epilogue warp: biases and groups of its 128 columns of the current tile
    alignas(16) float nb[K5_EPI_WARPS][K5_HALF];
    alignas(16) int grp[K5_EPI_WARPS][K5_HALF];
};
static_assert(offsetof(K5Ctl, nb) % 16 == 0 && offsetof(K5Ctl, grp) % 16 == 0,
              "float4 / int4 reads of the column data need 16-byte alignment");

struct K5Params {
    const ColInfo* col;  // [nc]
    float* numer;        // [b] diagonal logit, base-2 units
    float2* part;        // [chunks * 2][b] (running max, sum)
    int* err;
    int b, nc;
    float a2;            // log2(e) / tau
    int u_tiles;         // ceil(b / 128)
    int c_tiles;         // ceil(nc / 256)
    int chunks;          // column ranges (units = u_tiles * chunks)
    int kchunks;         // ceil(d / 64)
    int stages;
    uint32_t idesc;
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Column j's (bias bits, group); past nc: bias -inf and a group no row has.
__device__ __forceinline__ int2 load_col(const K5Params& p, int j) {
    if (j < p.nc) return __ldg(reinterpret_cast<const int2*>(p.col) + j);
    return make_int2((int)0xff800000u, -2);
}

__device__ __forceinline__ void unit_cols(const K5Params& p, int u, int* ut, int* ch, int* t0, int* t1) {
    *ut = u % p.u_tiles;
    *ch = u / p.u_tiles;
    *t0 = (int)((int64_t)p.c_tiles * *ch / p.chunks);
    *t1 = (int)((int64_t)p.c_tiles * (*ch + 1) / p.chunks);
}

// ---------------------------------------------------------------------------
// column preparation
// ---------------------------------------------------------------------------
__global__ void k5_table_clear(unsigned long long* keys, int64_t slots) {
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < slots;
         t += (int64_t)gridDim.x * blockDim.x)
        keys[t] = K5_EMPTY;
}

// Fibonacci hashing (Knuth, TAOCP vol. 3, 6.4): multiply by 2^64 / golden
// ratio and keep the top bits.
__device__ __forceinline__ int64_t k5_hash(unsigned long long id, int log2_slots) {
    return (int64_t)((id * 0x9E3779B97F4A7C15ull) >> (64 - log2_slots));
}

__global__ void k5_columns(const float* __restrict__ logq, const uint8_t* __restrict__ valid,
                           const int64_t* __restrict__ item_ids, int nc, unsigned long long* keys,
                           int log2_slots, ColInfo* __restrict__ col, int* err, unsigned* ticket) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j == 0) {
        *err = 0;
        *ticket = 0;
    }
    if (j >= nc) return;
    const float lq = logq ? logq[j] : 0.0f;
    const bool ok = valid ? valid[j] != 0 : true;
    ColInfo c;
    c.nb = ok ? -lq * K5_LOG2E : -INFINITY;
    c.g = 0;
    if (item_ids) {
        const unsigned long long id = (unsigned long long)item_ids[j];
        const int64_t slots = (int64_t)1 << log2_slots;
        if (id == K5_EMPTY) {
            c.g = (int)slots;  // the one id the table cannot hold has a group of its own
        } else {
            // linear probing; the table has at least twice as many slots as
            // columns, so a free or matching slot is always found
            int64_t h = k5_hash(id, log2_slots);
            for (int64_t probe = 0; probe < slots; ++probe) {
                const unsigned long long prev = atomicCAS(keys + h, K5_EMPTY, id);
                if (prev == K5_EMPTY || prev == id) {
                    c.g = (int)h;
                    break;
                }
                h = (h + 1) & (slots - 1);
            }
        }
    }
    col[j] = c;
}

// ---------------------------------------------------------------------------
// the fused scorer
// ---------------------------------------------------------------------------
template <bool HITS>
__global__ void __launch_bounds__(K5_THREADS, 1)
    k5_softmax(const __grid_constant__ CUtensorMap tm_users, const __grid_constant__ CUtensorMap tm_items,
               const K5Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* usm = smem;                                              // [kchunks][128 x 128 B]
    uint8_t* ring = smem + (size_t)p.kchunks * K5_USER_CHUNK;         // [stages][256 x 128 B]
    K5Ctl* ctl = reinterpret_cast<K5Ctl*>(ring + (size_t)p.stages * K5_STAGE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.u_tiles * p.chunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->ufull, 1);
        mbar_init(&ctl->uempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], K5_EPI_WARPS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, K5_TMEM_COLS);
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
            tma_prefetch_desc(&tm_users);
            tma_prefetch_desc(&tm_items);
            uint32_t it = 0;
            int uc = 0, u_issued = -1;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
                int ut, ch, t0, t1;
                unit_cols(p, u, &ut, &ch, &t0, &t1);
                if (!mbar_wait(&ctl->uempty, (uc & 1) ^ 1, abort)) { ok = false; break; }
                u_issued = uc;
                mbar_arrive_expect_tx(&ctl->ufull, (uint32_t)(p.kchunks * K5_USER_CHUNK));
                for (int kc = 0; kc < p.kchunks; ++kc)
                    tma_load_2d(usm + (size_t)kc * K5_USER_CHUNK, &tm_users, &ctl->ufull, kc * 64, ut * K5_M);
                for (int t = t0; ok && t < t1; ++t) {
                    for (int kc = 0; kc < p.kchunks; ++kc, ++it) {
                        const int s = it % p.stages;
                        if (!mbar_wait(&ctl->empty[s], ((it / p.stages) & 1) ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&ctl->full[s], K5_STAGE_BYTES);
                        tma_load_2d(ring + (size_t)s * K5_STAGE_BYTES, &tm_items, &ctl->full[s], kc * 64,
                                    t * K5_N);
                    }
                }
            }
            if (!ok) {
                atomicExch(p.err, ERR_TIMEOUT_TMA);
                *abort = 1;
            }
            // Every issued load must land before the block may exit.
            const uint32_t first = it > (uint32_t)p.stages ? it - p.stages : 0;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(&ctl->full[j % p.stages], (j / p.stages) & 1, nullptr);
            if (u_issued >= 0) mbar_wait(&ctl->ufull, u_issued & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            int uc = 0;
            bool ok = true;
            const uint32_t ubase = smem_u32(usm);
            const uint32_t rbase = smem_u32(ring);
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uc) {
                int ut, ch, t0, t1;
                unit_cols(p, u, &ut, &ch, &t0, &t1);
                if (!mbar_wait(&ctl->ufull, uc & 1, abort)) { ok = false; break; }
                tc_fence_after();
                for (int t = t0; ok && t < t1; ++t, ++tc) {
                    const int buf = tc & 1;
                    if (!mbar_wait(&ctl->tempty[buf], ((tc >> 1) & 1) ^ 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * K5_ACC_COLS);
                    for (int kc = 0; kc < p.kchunks; ++kc, ++it) {
                        const int s = it % p.stages;
                        if (!mbar_wait(&ctl->full[s], (it / p.stages) & 1, abort)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_addr = ubase + (uint32_t)(kc * K5_USER_CHUNK);
                        const uint32_t b_addr = rbase + (uint32_t)(s * K5_STAGE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // 16 bf16 (32 bytes) of K per MMA
                            umma_bf16(d_tmem, umma_desc_kmajor_sw128(a_addr + kk * 32),
                                      umma_desc_kmajor_sw128(b_addr + kk * 32), p.idesc,
                                      (kc | kk) != 0 ? 1u : 0u);
                        umma_commit(&ctl->empty[s]);  // stage free once these MMAs finish
                    }
                    if (ok) umma_commit(&ctl->tfull[buf]);  // accumulator ready
                }
                if (ok) umma_commit(&ctl->uempty);  // user tile free after this unit
            }
            if (!ok) {
                atomicExch(p.err, ERR_TIMEOUT_MMA);
                *abort = 1;
            }
            // Wait for every MMA issued by this thread before TMEM is freed.
            umma_commit(&ctl->drain);
            mbar_wait(&ctl->drain, 0, nullptr);
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        // Warp w reads TMEM lanes 32*(w%4).. (its 32 users) and one half of
        // the tile's 256 columns; each thread keeps (max, sum) for its user.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        float* nb_s = ctl->nb[ew];
        int* g_s = ctl->grp[ew];
        uint32_t tc = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            int ut, ch, t0, t1;
            unit_cols(p, u, &ut, &ch, &t0, &t1);
            const int i = ut * K5_M + quarter * 32 + lane;  // this thread's user
            const bool row_ok = i < p.b;
            const int my_g = (HITS && row_ok) ? p.col[i].g : -1;
            float m = K5_MAX_FLOOR;
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            for (int t = t0; t < t1; ++t, ++tc) {
                const int buf = tc & 1;
                const int jbase = t * K5_N + half * K5_HALF;
                // this warp's column data, fetched before waiting for the accumulator
                int2 ci0, ci1, ci2, ci3;  // (bias bits, group) of columns jbase + 32 e + lane
                ci0 = load_col(p, jbase + lane);
                ci1 = load_col(p, jbase + 32 + lane);
                ci2 = load_col(p, jbase + 64 + lane);
                ci3 = load_col(p, jbase + 96 + lane);
                __syncwarp();  // the previous tile's reads of nb_s / g_s are done
                nb_s[lane] = __int_as_float(ci0.x);
                nb_s[32 + lane] = __int_as_float(ci1.x);
                nb_s[64 + lane] = __int_as_float(ci2.x);
                nb_s[96 + lane] = __int_as_float(ci3.x);
                g_s[lane] = ci0.y;
                g_s[32 + lane] = ci1.y;
                g_s[64 + lane] = ci2.y;
                g_s[96 + lane] = ci3.y;
                __syncwarp();
                if (!mbar_wait(&ctl->tfull[buf], (tc >> 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                       (uint32_t)(buf * K5_ACC_COLS + half * K5_HALF);
#pragma unroll
                for (int pair = 0; pair < 2; ++pair) {
                    Cols32 v[2];
                    tmem_ld_32cols(tbase + (uint32_t)(2 * pair * 32), v[0].x);
                    tmem_ld_32cols(tbase + (uint32_t)((2 * pair + 1) * 32), v[1].x);
                    tmem_ld_wait();
                    if (pair == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->tempty[buf]);  // values are in registers now
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = 2 * pair + h;
                        const float4* nb4 = reinterpret_cast<const float4*>(nb_s + c * 32);
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 b4 = nb4[e4];
                            v[h].x[4 * e4 + 0] = fmaf(v[h].x[4 * e4 + 0], p.a2, b4.x);
                            v[h].x[4 * e4 + 1] = fmaf(v[h].x[4 * e4 + 1], p.a2, b4.y);
                            v[h].x[4 * e4 + 2] = fmaf(v[h].x[4 * e4 + 2], p.a2, b4.z);
                            v[h].x[4 * e4 + 3] = fmaf(v[h].x[4 * e4 + 3], p.a2, b4.w);
                        }
                        // the positive's logit, taken before the group test masks it
                        const int col0 = jbase + c * 32;
                        if (row_ok && (unsigned)(i - col0) < 32u) p.numer[i] = select32(v[h], i - col0);
                        if constexpr (HITS) {
                            const int4* g4 = reinterpret_cast<const int4*>(g_s + c * 32);
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const int4 gg = g4[e4];
                                if (gg.x == my_g) v[h].x[4 * e4 + 0] = -INFINITY;
                                if (gg.y == my_g) v[h].x[4 * e4 + 1] = -INFINITY;
                                if (gg.z == my_g) v[h].x[4 * e4 + 2] = -INFINITY;
                                if (gg.w == my_g) v[h].x[4 * e4 + 3] = -INFINITY;
                            }
                        }
                        float ca = v[h].x[0], cb = v[h].x[1];
#pragma unroll
                        for (int e = 2; e < 32; e += 4) {
                            ca = max3f(ca, v[h].x[e], v[h].x[e + 1]);
                            cb = max3f(cb, v[h].x[e + 2], v[h].x[e + 3]);
                        }
                        const float cmax = fmaxf(ca, cb);
                        if (cmax > m + K5_LAG) {  // raise the running max, rescale the sums
                            const float r = ex2_approx(m - cmax);
                            s0 *= r;
                            s1 *= r;
                            s2 *= r;
                            s3 *= r;
                            m = cmax;
                        }
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            s0 += ex2_approx(v[h].x[4 * e4 + 0] - m);
                            s1 += ex2_approx(v[h].x[4 * e4 + 1] - m);
                            s2 += ex2_approx(v[h].x[4 * e4 + 2] - m);
                            s3 += ex2_approx(v[h].x[4 * e4 + 3] - m);
                        }
                    }
                }
            }
            if (!ok) break;
            if (row_ok) p.part[(int64_t)(ch * 2 + half) * p.b + i] = make_float2(m, (s0 + s1) + (s2 + s3));
        }
        if (!ok) {
            atomicExch(p.err, ERR_TIMEOUT_EPI);
            *abort = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, K5_TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// merge: lse, loss, mean
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(K5_MERGE_THREADS)
    k5_merge(const float2* __restrict__ part, int parts, const float* __restrict__ numer,
             const uint8_t* __restrict__ valid, int b, int hits, const int* err, float* lse, float* loss,
             float* mean, double* block_sum, int* block_rows, unsigned* ticket) {
    __shared__ double red_s[K5_MERGE_THREADS / 32];
    __shared__ int red_n[K5_MERGE_THREADS / 32];
    __shared__ bool last;
    const int i = blockIdx.x * K5_MERGE_THREADS + threadIdx.x;
    const bool failed = *err != 0;
    double my_loss = 0.0;
    int my_rows = 0;
    if (i < b) {
        const float num = numer[i];
        float mx = hits ? num : -INFINITY;
        for (int q = 0; q < parts; ++q) mx = fmaxf(mx, part[(int64_t)q * b + i].x);
        float sum = hits && num != -INFINITY ? exp2f(num - mx) : 0.0f;
        for (int q = 0; q < parts; ++q) {
            const float2 pq = part[(int64_t)q * b + i];
            sum += pq.y * exp2f(pq.x - mx);
        }
        const float l2 = sum > 0.0f ? mx + log2f(sum) : -INFINITY;
        const bool row_valid = valid ? valid[i] != 0 : true;
        float li = row_valid ? (l2 - num) * K5_LN2 : 0.0f;
        float le = l2 * K5_LN2;
        if (failed) li = le = NAN;
        lse[i] = le;
        loss[i] = li;
        if (row_valid) {
            my_loss = (double)li;
            my_rows = 1;
        }
    }
    // block sums in a fixed order: warp shuffles, then the warps in order
    for (int o = 16; o > 0; o >>= 1) {
        my_loss += __shfl_xor_sync(0xffffffffu, my_loss, o);
        my_rows += __shfl_xor_sync(0xffffffffu, my_rows, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red_s[threadIdx.x >> 5] = my_loss;
        red_n[threadIdx.x >> 5] = my_rows;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        int n = 0;
        for (int w = 0; w < K5_MERGE_THREADS / 32; ++w) {
            s += red_s[w];
            n += red_n[w];
        }
        block_sum[blockIdx.x] = s;
        block_rows[blockIdx.x] = n;
        __threadfence();
        last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last && threadIdx.x == 0) {  // the last block adds the block sums in block order
        __threadfence();
        double s = 0.0;
        long long n = 0;
        for (unsigned blk = 0; blk < gridDim.x; ++blk) {
            s += ((volatile double*)block_sum)[blk];
            n += ((volatile int*)block_rows)[blk];
        }
        *mean = failed ? NAN : (n > 0 ? (float)(s / (double)n) : 0.0f);
    }
}

int softmax_stages(int d) {
    const int kchunks = (d + 63) / 64;
    const int fixed = 1024 + kchunks * K5_USER_CHUNK + (int)sizeof(K5Ctl);
    int stages = (K5_SMEM_BUDGET - fixed) / K5_STAGE_BYTES;
    if (stages > K5_MAX_STAGES) stages = K5_MAX_STAGES;
    return stages;
}

int log2_ceil(int64_t x) {
    int l = 0;
    while (((int64_t)1 << l) < x) ++l;
    return l;
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
SoftmaxPlan softmax_plan(int b, int nc, int d, bool item_ids, int sm_count) {
    SoftmaxPlan pl;
    pl.u_tiles = (b + K5_M - 1) / K5_M;
    pl.c_tiles = (nc + K5_N - 1) / K5_N;
    pl.stages = softmax_stages(d);
    // column ranges: make u_tiles * chunks a multiple of the SM count when
    // possible, else about four units per SM; at least one tile per range
    int chunks = 0;
    if (pl.u_tiles > 0) {
        for (int w = 1; w <= 8 && chunks == 0; ++w)
            if (((int64_t)sm_count * w) % pl.u_tiles == 0) chunks = (int)((int64_t)sm_count * w / pl.u_tiles);
        if (chunks == 0) chunks = (sm_count * 4 + pl.u_tiles - 1) / pl.u_tiles;
    }
    if (chunks < 1) chunks = 1;
    if (chunks > pl.c_tiles) chunks = pl.c_tiles > 0 ? pl.c_tiles : 1;
    pl.chunks = chunks;
    pl.log2_slots = item_ids ? log2_ceil(2 * (int64_t)(nc > 32 ? nc : 32)) : 0;
    pl.merge_blocks = (b + K5_MERGE_THREADS - 1) / K5_MERGE_THREADS;
    // workspace: every region starts on a 256-byte boundary
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    pl.off_err = take(sizeof(int));  // first: tt_inbatch_softmax_check reads it at offset 0
    pl.off_ticket = take(sizeof(unsigned));
    pl.off_col = take((size_t)nc * sizeof(ColInfo));
    pl.off_numer = take((size_t)b * sizeof(float));
    pl.off_part = take((size_t)chunks * 2 * b * sizeof(float2));
    pl.off_keys = take(item_ids ? ((size_t)1 << pl.log2_slots) * sizeof(unsigned long long) : 0);
    pl.off_block_sum = take((size_t)(pl.merge_blocks > 0 ? pl.merge_blocks : 1) * sizeof(double));
    pl.off_block_rows = take((size_t)(pl.merge_blocks > 0 ? pl.merge_blocks : 1) * sizeof(int));
    pl.bytes = off;
    return pl;
}

// d >= 64: every TMA box is 64 elements (128 bytes) of K wide.
bool softmax_supported(int d) { return d >= 64 && d <= 512 && softmax_stages(d) >= 2; }

cudaError_t launch_softmax(const SoftmaxPlan& pl, const CUtensorMap& tm_users, const CUtensorMap& tm_items,
                           int b, int nc, int d, float tau, const float* logq, const int64_t* item_ids,
                           const uint8_t* valid, float* lse, float* loss, float* mean, void* workspace,
                           cudaStream_t s, int sm_count) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    ColInfo* col = reinterpret_cast<ColInfo*>(ws + pl.off_col);
    float* numer = reinterpret_cast<float*>(ws + pl.off_numer);
    float2* part = reinterpret_cast<float2*>(ws + pl.off_part);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(ws + pl.off_keys);
    double* block_sum = reinterpret_cast<double*>(ws + pl.off_block_sum);
    int* block_rows = reinterpret_cast<int*>(ws + pl.off_block_rows);
    int* err = reinterpret_cast<int*>(ws + pl.off_err);
    unsigned* ticket = reinterpret_cast<unsigned*>(ws + pl.off_ticket);
    const bool hits = item_ids != nullptr;
    cudaError_t e;
    if (hits) {
        const int64_t slots = (int64_t)1 << pl.log2_slots;
        const int blocks = (int)((slots + 255) / 256 < 4 * sm_count ? (slots + 255) / 256 : 4 * sm_count);
        note_launch_begin(TT_KIND_SOFTMAX, s);
        k5_table_clear<<<blocks, 256, 0, s>>>(keys, slots);
        note_launch_end(TT_KIND_SOFTMAX, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    note_launch_begin(TT_KIND_SOFTMAX, s);
    k5_columns<<<(nc + 255) / 256 > 0 ? (nc + 255) / 256 : 1, 256, 0, s>>>(
        logq, valid, item_ids, nc, keys, pl.log2_slots, col, err, ticket);
    note_launch_end(TT_KIND_SOFTMAX, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (b == 0) return cudaMemsetAsync(mean, 0, sizeof(float), s);

    K5Params p;
    p.col = col;
    p.numer = numer;
    p.part = part;
    p.err = err;
    p.b = b;
    p.nc = nc;
    p.a2 = (float)(1.4426950408889634 / (double)tau);
    p.u_tiles = pl.u_tiles;
    p.c_tiles = pl.c_tiles;
    p.chunks = pl.chunks;
    p.kchunks = (d + 63) / 64;
    p.stages = pl.stages;
    p.idesc = umma_idesc_bf16(K5_M, K5_N);
    const int smem = 1024 + p.kchunks * K5_USER_CHUNK + p.stages * K5_STAGE_BYTES + (int)sizeof(K5Ctl);
    const int n_units = p.u_tiles * p.chunks;
    const int grid = n_units < sm_count ? n_units : sm_count;
    e = hits ? cudaFuncSetAttribute(k5_softmax<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
             : cudaFuncSetAttribute(k5_softmax<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    note_launch_begin(TT_KIND_SOFTMAX, s);
    if (hits)
        k5_softmax<true><<<grid, K5_THREADS, smem, s>>>(tm_users, tm_items, p);
    else
        k5_softmax<false><<<grid, K5_THREADS, smem, s>>>(tm_users, tm_items, p);
    note_launch_end(TT_KIND_SOFTMAX, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    note_launch_begin(TT_KIND_SOFTMAX, s);
    k5_merge<<<pl.merge_blocks, K5_MERGE_THREADS, 0, s>>>(part, pl.chunks * 2, numer, valid, b, hits ? 1 : 0,
                                                           err, lse, loss, mean, block_sum, block_rows, ticket);
    note_launch_end(TT_KIND_SOFTMAX, s);
    return cudaGetLastError();
}

}  // namespace tt
