// k_tensor_pair.cu - K3 for large query batches: the scoring contraction on
// pairs of SMs.
//
// Same product as the single-CTA tensor-core kernel (recsys_two_tower_model.py
// `forward` / `compute_top_k`: matmul(user.astype(bf16), post_embeddings.T)),
// with the same fused filter, but issued as paired tcgen05 MMAs
// (cta_group::2) by the two CTAs of a cluster, which sit on the two SMs of
// one TPC:
//
//   M = 256 queries   (128 in each CTA's shared memory, resident per unit)
//   N = 256 corpus rows (128 in each CTA's shared memory, streamed)
//   K = 16 per instruction, fp32 accumulators in tensor memory.
//
// Each CTA's tensor memory receives its own 128 queries (TMEM lanes) against
// all 256 corpus rows of the tile (TMEM columns). Against the single-CTA
// kernel (corpus rows on lanes, queries on columns) this
//   - reads 8 KB of operands from shared memory per SM and K step instead of
//     12 KB, which leaves shared-memory bandwidth for the TMA writes;
//   - gives every epilogue thread one query, so its threshold stays in
//     registers and the fast test is one compare per score with no
//     shared-memory traffic (with per-row norms the row scales are read once
//     per tile from shared memory).
//
// The epilogue reads its 128 accumulator columns with one TMEM round trip
// (four loads, one wait) and hands the accumulator back to the MMA issuer
// before testing anything: with d = 128 a tile is only eight MMAs long, and
// the hand-off is on the MMAs' critical path. A survivor of the exact test is
// staged in shared memory by its lane; the warp appends every lane's staged
// keys with one atomic instruction, so the lanes' round trips to the counters
// overlap instead of stalling the warp once per survivor.
//
// Roles (320 threads per CTA): warp 0 issues this CTA's TMA loads; warp 1
// allocates tensor memory (both CTAs) and, in the even CTA, issues the MMAs;
// warps 2..9 are the epilogue. Both CTAs' loads signal the even CTA's
// "stage full" barrier (paired TMA form, no multicast: each CTA loads only
// its own halves); stages and accumulators are handed back to both CTAs by
// multicast tcgen05.commit; the odd CTA's epilogue releases an accumulator
// with a remote mbarrier arrival.
//
// Every wait is bounded. On expiry a role records an error code and raises
// the abort flag of both CTAs; the kernel then drains its own copies and
// MMAs, meets the other CTA at a cluster barrier and frees tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int KP_QROWS = 128;                  // queries per CTA (M = 256 per pair)
constexpr int KP_ROWS = 128;                   // corpus rows per CTA and tile
constexpr int KP_TILE = 2 * KP_ROWS;           // corpus rows per tile (N)
constexpr int KP_KC = 64;                      // bf16 elements per 128-byte swizzle row
constexpr int KP_STAGE_BYTES = KP_ROWS * 128;  // one K chunk of this CTA's rows
constexpr int KP_QCHUNK_BYTES = KP_QROWS * 128;
constexpr int KP_MAX_STAGES = 12;
constexpr int KP_EPI_WARPS = 8;
constexpr int KP_THREADS = 32 * (2 + KP_EPI_WARPS);
constexpr int KP_TMEM_COLS = 512;
constexpr int KP_ACC_COLS = 256;
constexpr int KP_WARP_COLS = 128;              // columns (corpus rows) one epilogue warp reads
constexpr int KP_SMEM_BUDGET = 227 * 1024;
// Survivors a lane keeps in shared memory before the warp appends them to
// the global lists with one atomic instruction for all its lanes.
constexpr int KP_STAGED = 8;

struct KPCtl {
    uint64_t full[KP_MAX_STAGES];    // even CTA: both CTAs' halves of the stage landed
    uint64_t empty[KP_MAX_STAGES];   // stage consumed (multicast commit)
    uint64_t qfull, qempty;          // query tiles: landed (even CTA) / consumed
    uint64_t tfull[2];               // accumulator ready (multicast commit)
    uint64_t tempty[2];              // even CTA: accumulator drained by both epilogues
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    // per-row score scales (rows with norms), read as float4
    alignas(16) float cvals[KP_EPI_WARPS][KP_WARP_COLS];
    // per epilogue lane: survivors waiting for their append ([slot][lane])
    uint64_t staged[KP_EPI_WARPS][KP_STAGED][32];
    // int8: per epilogue thread, its query's scale and score floor (kept out
    // of registers: ten warps leave 168 registers per thread)
    float q_us[KP_EPI_WARPS][32];
    float q_t[KP_EPI_WARPS][32];
};
static_assert(offsetof(KPCtl, cvals) % 16 == 0, "float4 reads of cvals need 16-byte alignment");

struct KPParams {
    PassArgs a;
    int q_tiles;    // ceil(b / 256)
    int kchunks;    // ceil(d / 64)
    int kps;        // K chunks per ring stage
    int stages;
    int64_t tiles;  // corpus tiles of 256 rows in this level
    int chunks;     // corpus chunks (units = q_tiles * chunks)
    uint32_t idesc;
};

__device__ __forceinline__ void unit_range(const KPParams& p, int u, int* qt, int64_t* t0,
                                           int64_t* t1) {
    *qt = u % p.q_tiles;
    const int ch = u / p.q_tiles;
    *t0 = p.tiles * ch / p.chunks;
    *t1 = p.tiles * (ch + 1) / p.chunks;
}

// Raise the abort flag in both CTAs of the pair.
__device__ __forceinline__ void raise_abort(KPCtl* ctl, uint32_t peer) {
    ctl->abort = 1;
    st_cluster_u32(mapa_shared(&ctl->abort, peer), 1u);
}

// NORMS: per-row score scales (raw rows with norms); MASK: an exclusion
// bitmask; TYPES: several result sets by candidate type; I8: int8 codes
// (kind::i8, int32 accumulators) with per-row and per-query scales.
template <bool NORMS, bool MASK, bool TYPES, bool I8, int KPS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(KP_THREADS, 1)
    k3_pair(const __grid_constant__ CUtensorMap tm_rows, const __grid_constant__ CUtensorMap tm_q,
            const KPParams p) {
    static_assert(!(I8 && (NORMS || TYPES)), "int8 rows carry their scales themselves");
    constexpr int KC = I8 ? 128 : KP_KC;  // elements per 128-byte swizzle row
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* qsm = smem;                                          // [kchunks][128 x 128 B]
    uint8_t* ring = smem + (size_t)p.kchunks * KP_QCHUNK_BYTES;   // [stages][16 KB]
    KPCtl* ctl = reinterpret_cast<KPCtl*>(ring + (size_t)p.stages * KPS * KP_STAGE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const bool even = rank == 0;
    const int cid = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;
    const int n_units = p.q_tiles * p.chunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->qfull, 1);
        mbar_init(&ctl->qempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * KP_EPI_WARPS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_base, KP_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int* abort = &ctl->abort;

    if (warp == 0) {
        // ---------------------------- TMA producer (both CTAs) ----------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_rows);
            tma_prefetch_desc(&tm_q);
            // Both CTAs' copies complete on the even CTA's barriers; the even
            // CTA's producer announces the bytes of both halves.
            const uint32_t qfull0 = mapa_shared(&ctl->qfull, 0);
            uint32_t it = 0;
            int uc = 0, q_issued = -1;
            bool ok = true;
            for (int u = cid; ok && u < n_units; u += n_clusters, ++uc) {
                int qt;
                int64_t t0, t1;
                unit_range(p, u, &qt, &t0, &t1);
                if (!mbar_wait(&ctl->qempty, (uc & 1) ^ 1, abort)) { ok = false; break; }
                q_issued = uc;
                if (even) mbar_arrive_expect_tx(&ctl->qfull, (uint32_t)(2 * p.kchunks * KP_QCHUNK_BYTES));
                for (int kc = 0; kc < p.kchunks; ++kc)
                    tma_load_2d_pair(qsm + (size_t)kc * KP_QCHUNK_BYTES, &tm_q, qfull0, kc * KC,
                                     qt * (2 * KP_QROWS) + (int)rank * KP_QROWS);
                for (int64_t t = t0; ok && t < t1; ++t) {
                    for (int kg = 0; kg < p.kchunks; kg += KPS, ++it) {
                        const int s = it % p.stages;
                        if (!mbar_wait(&ctl->empty[s], ((it / p.stages) & 1) ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        if (even) mbar_arrive_expect_tx(&ctl->full[s], (uint32_t)(2 * KPS * KP_STAGE_BYTES));
#pragma unroll
                        for (int j = 0; j < KPS; ++j)
                            tma_load_2d_pair(ring + ((size_t)s * KPS + j) * KP_STAGE_BYTES, &tm_rows,
                                             mapa_shared(&ctl->full[s], 0), (kg + j) * KC,
                                             (int32_t)(t * KP_TILE + (int64_t)rank * KP_ROWS));
                    }
                }
            }
            if (!ok) {
                atomicExch(p.a.err, ERR_TIMEOUT_TMA);
                raise_abort(ctl, peer);
            }
            // Every load of the pair must land before either CTA may exit: the
            // even CTA waits for the last phases of its barriers (which count
            // both halves), and the odd CTA waits for the even one at the
            // final cluster barrier. After an abort a phase may lack the other
            // CTA's half, hence the short limit.
            if (even) {
                const unsigned long long drain_ns = 20000000ull;
                const uint32_t first = it > (uint32_t)p.stages ? it - p.stages : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&ctl->full[j % p.stages], (j / p.stages) & 1, nullptr, drain_ns);
                if (q_issued >= 0) mbar_wait(&ctl->qfull, q_issued & 1, nullptr, drain_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && even) {
            // ------------------------ MMA issuer (even CTA) ------------------------
            uint32_t it = 0, tc = 0;
            int uc = 0;
            bool ok = true;
            const uint32_t qbase = smem_u32(qsm);
            const uint32_t rbase = smem_u32(ring);
            for (int u = cid; ok && u < n_units; u += n_clusters, ++uc) {
                int qt;
                int64_t t0, t1;
                unit_range(p, u, &qt, &t0, &t1);
                if (!mbar_wait_cluster(&ctl->qfull, uc & 1, abort)) { ok = false; break; }
                tc_fence_after();
                for (int64_t t = t0; ok && t < t1; ++t, ++tc) {
                    const int buf = tc & 1;
                    if (!mbar_wait_cluster(&ctl->tempty[buf], ((tc >> 1) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * KP_ACC_COLS);
                    for (int kg = 0; kg < p.kchunks; kg += KPS, ++it) {
                        const int s = it % p.stages;
                        const uint32_t par = (it / p.stages) & 1;
                        if (!mbar_wait_cluster(&ctl->full[s], par, abort)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int j = 0; j < KPS; ++j) {
                            const int kc = kg + j;
                            const uint32_t a_addr = qbase + (uint32_t)(kc * KP_QCHUNK_BYTES);
                            const uint32_t b_addr = rbase + (uint32_t)((s * KPS + j) * KP_STAGE_BYTES);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {  // 32 bytes of K per instruction
                                if constexpr (I8)
                                    umma_i8_pair(d_tmem, umma_desc_kmajor_sw128(a_addr + kk * 32),
                                                 umma_desc_kmajor_sw128(b_addr + kk * 32), p.idesc,
                                                 (kc | kk) != 0 ? 1u : 0u);
                                else
                                    umma_bf16_pair(d_tmem, umma_desc_kmajor_sw128(a_addr + kk * 32),
                                                   umma_desc_kmajor_sw128(b_addr + kk * 32), p.idesc,
                                                   (kc | kk) != 0 ? 1u : 0u);
                            }
                        }
                        umma_commit_pair_mc(&ctl->empty[s], 0x3);  // stage free in both CTAs
                    }
                    if (ok) umma_commit_pair_mc(&ctl->tfull[buf], 0x3);  // accumulator ready
                }
                if (ok) umma_commit_pair_mc(&ctl->qempty, 0x3);  // query tiles free
            }
            if (!ok) {
                atomicExch(p.a.err, ERR_TIMEOUT_MMA);
                raise_abort(ctl, peer);
            }
            // Every MMA issued here must finish before tensor memory is freed.
            umma_commit_pair(&ctl->drain);
            mbar_wait(&ctl->drain, 0, nullptr);
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        // Warp w reads TMEM lanes 32*(w%4).. (32 queries, one per thread) and
        // columns [128*half, 128*half + 128) of the accumulator (128 corpus rows).
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const PassArgs& a = p.a;
        float* cw = ctl->cvals[ew];
        uint64_t* staged = &ctl->staged[ew][0][lane];
        const uint32_t r_tempty0 = mapa_shared(&ctl->tempty[0], 0);
        const uint32_t r_tempty1 = mapa_shared(&ctl->tempty[1], 0);
        uint32_t tc = 0;
        bool ok = true;
        for (int u = cid; ok && u < n_units; u += n_clusters) {
            int qt;
            int64_t t0, t1;
            unit_range(p, u, &qt, &t0, &t1);
            // This thread's query and its thresholds (padding queries carry
            // KEY_MAX / +inf and never pass).
            const int q = qt * (2 * KP_QROWS) + (int)rank * KP_QROWS + quarter * 32 + lane;
            const uint64_t th_key = __ldg(a.theta + q);
            float t_fast = __ldg(a.thf + q);
            // int8: score = fl(fl(acc * us) * c_row); us is this thread's query scale
            if (I8) {
                // int8 fast test: a non-negative int32 accumulator below 2^23
                // (|code| <= 127, d <= 512), read as float bits, is the
                // subnormal acc * 2^-149, exactly; times c_row * 2^64 it gives
                // acc * c_row * 2^-85 with one rounding, a normal float for
                // scores near any threshold. A score fl(fl(acc * us) * c_row)
                // >= t > 0 needs acc * c_row >= t / us * (1 - 2^-23), so
                // t_fast = (t / us) * 2^-85 lowered by a relative 2^-20 (and
                // an absolute 2^-148 for the subnormal range) keeps every such
                // row. Negative accumulators read as negative floats or NaN,
                // and never reach a positive threshold. Without a positive
                // floor every score takes the exact test (t_fast = -inf, and
                // the test passes NaN maxima).
                const float us = q < a.b ? __ldg(a.qscale + q) : 1.0f;
                ctl->q_us[ew][lane] = us;
                ctl->q_t[ew][lane] = t_fast;
                if (!(t_fast > 0.0f)) {
                    t_fast = -INFINITY;
                } else if (t_fast != INFINITY) {
                    const float r = (t_fast / us) * 0x1p-85f;
                    t_fast = r - r * 0x1p-20f - 0x1p-148f;
                }
            }
            float neg_t_low = -t_fast;
            if (NORMS && t_fast != INFINITY && t_fast != -INFINITY)
                neg_t_low = -(t_fast - fabsf(t_fast) * 0x1p-20f - 0x1p-140f);
            uint32_t* cnt = a.count + q;
            uint64_t* qkeys = a.keys + (int64_t)q * a.cap;
            // Survivors are staged per lane and appended by the whole warp at
            // once: one atomic instruction reserves every lane's slots, so the
            // round trips of the 32 lanes overlap instead of stalling the warp
            // once per survivor.
            int n_staged = 0;
            auto flush = [&]() {
                const uint32_t base = n_staged > 0 ? atomicAdd(cnt, (uint32_t)n_staged) : 0u;
                for (int j = 0; j < n_staged; ++j)
                    if (base + j < (uint32_t)a.cap) qkeys[base + j] = staged[j * 32];
                n_staged = 0;
            };
            // Per-row data of this warp's 128 columns of a tile, fetched one
            // tile ahead: lane l holds rows l, l+32, l+64, l+96 - the inverse
            // norm (rows with norms; 0 past the last row), the mask word
            // holding the row's exclusion bit and that bit's position.
            float cl[4];
            uint32_t xl[4], xs[4];
            auto fetch_rows = [&](int64_t tile) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t r = tile * KP_TILE + half * KP_WARP_COLS + lane + 32 * j;
                    const bool valid = r < a.n_rows;
                    // raw values: nothing waits for these loads until the next tile
                    if (NORMS || I8) cl[j] = valid ? __ldg(a.inv_norm + r * a.stride) : 0.0f;
                    if (MASK) {
                        xl[j] = valid ? __ldg(a.exclude + ((r * a.stride) >> 5)) : 0u;
                        xs[j] = (uint32_t)((r * a.stride) & 31);
                    }
                }
            };
            if (NORMS || MASK || I8) fetch_rows(t0);
            for (int64_t t = t0; t < t1; ++t, ++tc) {
                const int buf = tc & 1;
                const int64_t row0 = t * KP_TILE + half * KP_WARP_COLS;  // level row of column 0
                // bit i of skip[j]: row row0 + 32j + i is excluded or past the end
                uint32_t skip[4] = {0u, 0u, 0u, 0u};
                if (MASK || row0 + KP_WARP_COLS > a.n_rows) {  // warp-uniform
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        bool bad = row0 + lane + 32 * j >= a.n_rows;
                        if (MASK) bad |= ((xl[j] >> xs[j]) & 1u) != 0u;
                        skip[j] = __ballot_sync(0xFFFFFFFFu, bad);
                    }
                }
                if (NORMS || I8) {
                    __syncwarp();  // the previous tile's reads of cw are done
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        cw[lane + 32 * j] = I8 ? (cl[j] * a.inv_tau) * 0x1p64f : cl[j] * a.inv_tau;
                    __syncwarp();
                }
                if ((NORMS || MASK || I8) && t + 1 < t1) fetch_rows(t + 1);
                // the warp decides together, so that it stays converged
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ctl->tfull[buf], (tc >> 1) & 1, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                       (uint32_t)(buf * KP_ACC_COLS + half * KP_WARP_COLS);
                // One round trip: the warp's 128 columns into registers, then
                // the accumulator goes back to the MMA issuer before any test.
                // (int8 and rows with norms: two round trips of 64 columns, the
                // accumulator going back after the second; their fast tests
                // need the registers - with four chunks held the norms variant
                // spilled and ran 45 % slower.)
                constexpr int NV = (I8 || NORMS) ? 2 : 4;  // 32-column chunks held at once
#pragma unroll
                for (int part = 0; part < 4 / NV; ++part) {
                Cols32 v[NV];
#pragma unroll
                for (int h = 0; h < NV; ++h) tmem_ld_32cols(tbase + (uint32_t)((part * NV + h) * 32), v[h].x);
                tmem_ld_wait();
                if (part == 4 / NV - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (even)
                            mbar_arrive(&ctl->tempty[buf]);
                        else
                            mbar_arrive_cluster_relaxed(buf ? r_tempty1 : r_tempty0);
                    }
                }
#pragma unroll
                for (int h = 0; h < NV; ++h) {
                    const int hc = part * NV + h;  // chunk of the warp's 128 columns
                    const int col0 = hc * 32;      // within this warp's 128 columns
                    // Fast test. One threshold per thread: compare the maximum
                    // of the 32 scores (four chains of three-input max, half an
                    // instruction per score).
                    bool pass;
                    float gmax[4];
                    if (I8) {
                        const float* cc = cw + col0;  // c_row * 2^64 (one broadcast read per score)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {  // chain j: scores 8j .. 8j+7
                            const float* x = v[h].x + 8 * j;
                            const float* c = cc + 8 * j;
                            gmax[j] = fmaxf(max3f(max3f(max3f(x[0] * c[0], x[1] * c[1], x[2] * c[2]), x[3] * c[3],
                                                        x[4] * c[4]),
                                                  x[5] * c[5], x[6] * c[6]),
                                            x[7] * c[7]);
                        }
                        pass = !(fmaxf(max3f(gmax[0], gmax[1], gmax[2]), gmax[3]) < t_fast);
                    } else if (!NORMS) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {  // chain j: scores 8j .. 8j+7
                            const float* x = v[h].x + 8 * j;
                            gmax[j] = fmaxf(max3f(max3f(max3f(x[0], x[1], x[2]), x[3], x[4]), x[5], x[6]), x[7]);
                        }
                        pass = fmaxf(max3f(gmax[0], gmax[1], gmax[2]), gmax[3]) >= t_fast;
                    } else {
                        // all-negative test: AND of the sign words
                        const float4* c4 = reinterpret_cast<const float4*>(cw + col0);
                        uint32_t n0 = ~0u, n1 = ~0u;
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 c = c4[i4];
                            n0 &= __float_as_uint(fmaf(v[h].x[4 * i4 + 0], c.x, neg_t_low)) &
                                  __float_as_uint(fmaf(v[h].x[4 * i4 + 1], c.y, neg_t_low));
                            n1 &= __float_as_uint(fmaf(v[h].x[4 * i4 + 2], c.z, neg_t_low)) &
                                  __float_as_uint(fmaf(v[h].x[4 * i4 + 3], c.w, neg_t_low));
                        }
                        pass = ((n0 & n1) >> 31) == 0u;
                    }
                    if (!pass) continue;
                    // Rare: this thread's exact survivors among the 32 rows.
                    uint32_t m = 0;
                    if (I8) {
                        // exact scores, only in the groups of eight whose
                        // maximum passed (acc is exact in fp32: |acc| < 2^24)
                        const float us = ctl->q_us[ew][lane], t_exact = ctl->q_t[ew][lane];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (!(gmax[j] < t_fast)) {
#pragma unroll
                                for (int i = 8 * j; i < 8 * j + 8; ++i)
                                    m |= ((float)__float_as_int(v[h].x[i]) * us * (cw[col0 + i] * 0x1p-64f) >= t_exact)
                                             ? (1u << i) : 0u;
                            }
                        }
                    } else if (!NORMS) {
                        // only the groups of eight whose maximum passed
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (gmax[j] >= t_fast) {
#pragma unroll
                                for (int i = 8 * j; i < 8 * j + 8; ++i) m |= (v[h].x[i] >= t_fast) ? (1u << i) : 0u;
                            }
                        }
                    } else {
                        const float4* c4 = reinterpret_cast<const float4*>(cw + col0);
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 c = c4[i4];
                            m |= (v[h].x[4 * i4 + 0] * c.x >= t_fast) ? (1u << (4 * i4 + 0)) : 0u;
                            m |= (v[h].x[4 * i4 + 1] * c.y >= t_fast) ? (1u << (4 * i4 + 1)) : 0u;
                            m |= (v[h].x[4 * i4 + 2] * c.z >= t_fast) ? (1u << (4 * i4 + 2)) : 0u;
                            m |= (v[h].x[4 * i4 + 3] * c.w >= t_fast) ? (1u << (4 * i4 + 3)) : 0u;
                        }
                    }
                    m &= ~skip[hc];
                    while (m) {
                        const int i = __ffs(m) - 1;
                        m &= m - 1;
                        const int64_t id = (row0 + col0 + i) * a.stride;
                        const float c = NORMS ? cw[col0 + i] : a.inv_tau;
                        const float sc = I8 ? (float)__float_as_int(select32(v[h], i)) * ctl->q_us[ew][lane] *
                                                  (cw[col0 + i] * 0x1p-64f)
                                            : select32(v[h], i) * c;
                        const uint64_t key = make_key(sc, (uint32_t)id);
                        if (TYPES) {  // several result sets: the row's set, appended at once
                            const int rset = a.set_of[a.types[id]];
                            if (rset >= 0 && q < a.b) {
                                const int64_t vq = (int64_t)rset * a.b + q;
                                if (key > a.theta_v[vq]) {
                                    const uint32_t slot = atomicAdd(a.count + vq, 1u);
                                    if (slot < (uint32_t)a.cap) a.keys[vq * a.cap + slot] = key;
                                }
                            }
                        } else if (key > th_key) {
                            if (n_staged < KP_STAGED) {
                                staged[n_staged * 32] = key;
                                ++n_staged;
                            } else {  // this lane's staging is full: append on its own
                                const uint32_t slot = atomicAdd(cnt, 1u);
                                if (slot < (uint32_t)a.cap) qkeys[slot] = key;
                            }
                        }
                    }
                }
                }  // part
                if (!TYPES && __any_sync(0xFFFFFFFFu, n_staged >= KP_STAGED / 2)) flush();
            }
            if (!TYPES && __any_sync(0xFFFFFFFFu, n_staged > 0)) flush();
        }
        if (!ok) {
            atomicExch(a.err, ERR_TIMEOUT_EPI);
            raise_abort(ctl, peer);
        }
    }

    tc_fence_before();
    __syncthreads();
    // Neither CTA may exit or free tensor memory while the pair's MMAs, remote
    // arrivals or multicast commits can still reach it.
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, KP_TMEM_COLS);
    }
}

// K chunks of 128 bytes per row: 64 bf16 or 128 int8 elements each.
int pair_kchunks(int d, int esize) { return (d * esize + 127) / 128; }

// K chunks per ring stage: two for rows of two chunks (d = 128 bf16: one
// barrier handshake and one commit per tile), else one (the single-SM kernel
// measured slower with two on rows of four chunks).
int pair_kps(int kchunks) { return kchunks == 2 ? 2 : 1; }

int pair_stages(int d, int esize) {
    const int kchunks = pair_kchunks(d, esize);
    const int fixed = 1024 + kchunks * KP_QCHUNK_BYTES + (int)sizeof(KPCtl);
    int stages = (KP_SMEM_BUDGET - fixed) / (pair_kps(kchunks) * KP_STAGE_BYTES);
    if (stages > KP_MAX_STAGES) stages = KP_MAX_STAGES;
    return stages;
}

template <bool NORMS, bool MASK, bool TYPES, bool I8 = false>
cudaError_t launch_variant(const KPParams& base, const CUtensorMap& tm_rows, const CUtensorMap& tm_queries,
                           int smem, cudaStream_t s, int sm_count) {
    // the stage grouping is a compile-time constant: a run-time bound on the
    // MMA issuer's inner loop cost the single-SM kernel 8 % on 2*10^7 x 256 rows
    auto kern = base.kps == 2 ? k3_pair<NORMS, MASK, TYPES, I8, 2> : k3_pair<NORMS, MASK, TYPES, I8, 1>;
    KPParams p = base;
    // Pairs that can be resident at once (clusters must fit inside a GPC).
    int pairs = sm_count / 2 > 0 ? sm_count / 2 : 1;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * pairs);
        cfg.blockDim = dim3(KP_THREADS);
        cfg.dynamicSmemBytes = (size_t)smem;
        int max_clusters = 0;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) == cudaSuccess) {
            if (max_clusters > 0 && max_clusters < pairs) pairs = max_clusters;
        } else {
            cudaGetLastError();
        }
    }
    // Corpus chunks: make q_tiles * chunks a multiple of the number of pairs
    // when possible (every pair gets the same number of units).
    int chunks = 0;
    for (int w = 1; w <= 8 && chunks == 0; ++w)
        if (((int64_t)pairs * w) % p.q_tiles == 0) chunks = (int)((int64_t)pairs * w / p.q_tiles);
    if (chunks == 0) chunks = (pairs * 4 + p.q_tiles - 1) / p.q_tiles;
    if (chunks < 1) chunks = 1;
    if (chunks > p.tiles) chunks = (int)p.tiles;
    p.chunks = chunks;
    const int n_units = p.q_tiles * p.chunks;
    const int clusters = n_units < pairs ? n_units : pairs;
    note_launch_begin(TT_KIND_TENSOR, s);
    kern<<<2 * clusters, KP_THREADS, smem, s>>>(tm_rows, tm_queries, p);
    note_launch_end(TT_KIND_TENSOR, s);
    return cudaGetLastError();
}

}  // namespace

int tensor_pair_box_rows(int) { return KP_ROWS; }

int tensor_pair_smem_bytes(int d, int esize) {
    if (d > TT_MAX_D) return -1;
    const int kchunks = pair_kchunks(d, esize);
    const int stages = pair_stages(d, esize);
    if (stages < 2) return -1;
    return 1024 + kchunks * KP_QCHUNK_BYTES + (int)sizeof(KPCtl) + stages * pair_kps(kchunks) * KP_STAGE_BYTES;
}

cudaError_t launch_tensor_pair_pass(const PassArgs& a, const CUtensorMap& tm_rows, cudaStream_t s, int sm_count) {
    if (a.n_rows == 0 || a.b == 0) return cudaSuccess;
    const bool i8 = a.dtype == TT_I8;
    if (a.q_dtype != (i8 ? TT_I8 : TT_BF16)) return cudaErrorInvalidValue;
    if (i8 && (a.types != nullptr || a.inv_norm == nullptr || a.qscale == nullptr)) return cudaErrorInvalidValue;
    const int esize = i8 ? 1 : 2;
    const int smem = tensor_pair_smem_bytes(a.d, esize);
    if (smem <= 0) return cudaErrorInvalidValue;
    CUtensorMap tm_queries;
    const bool mapped = i8 ? i8_tile_tensor_map(a.queries, a.b, a.d, a.d, KP_QROWS, &tm_queries)
                           : bf16_tile_tensor_map(a.queries, a.b, a.d, a.d, KP_QROWS, &tm_queries);
    if (!mapped) return cudaErrorInvalidValue;
    KPParams p;
    p.a = a;
    p.q_tiles = (a.b + 2 * KP_QROWS - 1) / (2 * KP_QROWS);
    p.kchunks = pair_kchunks(a.d, esize);
    p.kps = pair_kps(p.kchunks);
    p.stages = pair_stages(a.d, esize);
    p.tiles = (a.n_rows + KP_TILE - 1) / KP_TILE;
    p.chunks = 1;
    p.idesc = i8 ? umma_idesc_s8(2 * KP_QROWS, KP_TILE) : umma_idesc_bf16(2 * KP_QROWS, KP_TILE);
    const bool norms = a.inv_norm != nullptr, mask = a.exclude != nullptr, types = a.types != nullptr;
    if (i8)  // the row scales go through the int8 epilogue, not the norms one
        return mask ? launch_variant<false, true, false, true>(p, tm_rows, tm_queries, smem, s, sm_count)
                    : launch_variant<false, false, false, true>(p, tm_rows, tm_queries, smem, s, sm_count);
    if (types) {
        return norms ? launch_variant<true, true, true>(p, tm_rows, tm_queries, smem, s, sm_count)
                     : launch_variant<false, true, true>(p, tm_rows, tm_queries, smem, s, sm_count);
    }
    if (norms)
        return mask ? launch_variant<true, true, false>(p, tm_rows, tm_queries, smem, s, sm_count)
                    : launch_variant<true, false, false>(p, tm_rows, tm_queries, smem, s, sm_count);
    return mask ? launch_variant<false, true, false>(p, tm_rows, tm_queries, smem, s, sm_count)
                : launch_variant<false, false, false>(p, tm_rows, tm_queries, smem, s, sm_count);
}

}  // namespace tt
