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
//   k5_sort_count,  (with item ids) a stable counting sort of the rows and of
//   k5_sort_scan,   the columns by a 256-bin hash of the item id (rows and the
//   k5_sort_scatter first b columns by one permutation, the shared negatives
//   k5_permute      by another), then copies of the users, the items and the
//                   column data in that order, so that a row's hits can only lie
//                   in its bins' column ranges
//   k5_softmax      tcgen05 MMAs of 128 users x 192 candidates into TMEM;
//                   the epilogue turns each accumulator row into running
//                   (max, sum of 2^(x - max)) pairs, x = acc * log2(e)/tau + nb_j,
//                   so the exponentials never leave registers
//   k5_merge        per row: combine the partial pairs (and, with item ids,
//                   the diagonal term the group test left out), lse, loss
//                   (written at the row's own index), and the mean over valid
//                   rows in a fixed order
//
// The epilogue runs in base-2 units so that each term is one ex2.approx
// (MUFU) instruction; that unit, 16 results per clock per SM, bounds the
// kernel at d <= 128, not the tensor cores. With item ids, the hit test (a
// compare and a select per logit) would cost as much issue time as the
// exponential itself; in the bin order, an epilogue warp's 32 rows fall in a
// few bins, so one warp-uniform range test per 32-column chunk tells where a
// hit is possible at all and only those chunks (a few percent) run the test.
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
constexpr int K5_N = 192;                    // candidates per tile (TMEM columns, <= K5_ACC_COLS)
constexpr int K5_USER_CHUNK = K5_M * 128;    // one 128-byte K chunk of the user tile
constexpr int K5_STAGE_BYTES = K5_N * 128;   // one 128-byte K chunk of a candidate tile
constexpr int K5_MAX_STAGES = 8;
constexpr int K5_EPI_WARPS = 12;              // 4 TMEM lane quarters x K5_COL_GROUPS
constexpr int K5_COL_GROUPS = K5_EPI_WARPS / 4;
constexpr int K5_WARP_COLS = K5_N / K5_COL_GROUPS;  // columns of one epilogue warp
constexpr int K5_WARP_CHUNKS = K5_WARP_COLS / 32;   // 32-column TMEM loads per warp and tile
static_assert(K5_EPI_WARPS % 4 == 0 && K5_WARP_CHUNKS % 2 == 0 && K5_WARP_COLS * K5_COL_GROUPS == K5_N,
              "epilogue split");
constexpr int K5_THREADS = 32 * (2 + K5_EPI_WARPS);
constexpr int K5_TMEM_COLS = 512;
constexpr int K5_ACC_COLS = 256;
constexpr int K5_SMEM_BUDGET = 227 * 1024;
constexpr float K5_MAX_FLOOR = -1e30f;       // running max before any column (base-2 units)
constexpr float K5_SUM_LIMIT = 0x1p64f;      // largest chunk sum taken without raising the max
constexpr float K5_LOG2E = 1.4426950408889634f;
constexpr float K5_LN2 = 0.6931471805599453f;
constexpr unsigned long long K5_EMPTY = 0x8000000000000000ull;  // free table slot
constexpr int K5_MERGE_THREADS = 256;
constexpr int K5_BINS = 256;                 // sort bins: the top 8 bits of the id's hash
constexpr int K5_SORT_THREADS = 256;         // one element per thread and round
constexpr int K5_SORT_WARPS = K5_SORT_THREADS / 32;
constexpr int K5_SCAN_THREADS = 1024;
static_assert(K5_SORT_THREADS == K5_BINS, "the bin-order kernels give each thread one bin");
static_assert(K5_SORT_THREADS % 32 == 0, "whole warps: the scatter matches bins across all 32 lanes");

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
    // per epilogue warp: biases and groups of its columns, for two tiles in flight
    alignas(16) float nb[K5_EPI_WARPS][2][K5_WARP_COLS];
    alignas(16) int grp[K5_EPI_WARPS][2][K5_WARP_COLS];
    // per epilogue warp, with item ids: the column ranges [lo0, hi0) and
    // [lo1, hi1) where its rows can have hits (kept here, not in registers)
    alignas(16) int hit_cols[K5_EPI_WARPS][4];
};
static_assert(offsetof(K5Ctl, nb) % 16 == 0 && offsetof(K5Ctl, grp) % 16 == 0,
              "float4 / int4 reads of the column data need 16-byte alignment");

struct K5Params {
    const ColInfo* col;  // [nc] (with item ids: in the bin order)
    const uint8_t* sbin; // with item ids: [b] bin of each row in the bin order, else null
    const int* bstart;   // with item ids: [2][K5_BINS + 1] first column of each bin, in-batch
                         // columns then shared negatives (the last entry: the part's end)
    float* numer;        // [b] diagonal logit, base-2 units
    float2* part;        // [chunks * K5_COL_GROUPS][b] (running max, sum)
    int* err;
    int b, nc;
    float a2;            // log2(e) / tau
    int u_tiles;         // ceil(b / 128)
    int c_tiles;         // ceil(nc / K5_N)
    int chunks;          // column ranges (units = u_tiles * chunks)
    int kchunks;         // ceil(d / 64)
    int stages;
    uint32_t idesc;
};

// Packed fp32 pairs (sm_100 f32x2): two lanes of work per instruction.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Keep the compiler from moving uses of TMEM-loaded registers above the
// tcgen05.wait::ld that makes them valid.
__device__ __forceinline__ void fence_regs(Cols32& c) {
    asm volatile(""
                 : "+f"(c.x[0]), "+f"(c.x[1]), "+f"(c.x[2]), "+f"(c.x[3]), "+f"(c.x[4]), "+f"(c.x[5]),
                   "+f"(c.x[6]), "+f"(c.x[7]), "+f"(c.x[8]), "+f"(c.x[9]), "+f"(c.x[10]), "+f"(c.x[11]),
                   "+f"(c.x[12]), "+f"(c.x[13]), "+f"(c.x[14]), "+f"(c.x[15]), "+f"(c.x[16]), "+f"(c.x[17]),
                   "+f"(c.x[18]), "+f"(c.x[19]), "+f"(c.x[20]), "+f"(c.x[21]), "+f"(c.x[22]), "+f"(c.x[23]),
                   "+f"(c.x[24]), "+f"(c.x[25]), "+f"(c.x[26]), "+f"(c.x[27]), "+f"(c.x[28]), "+f"(c.x[29]),
                   "+f"(c.x[30]), "+f"(c.x[31]));
}

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
// the bin order (item ids only)
//
// A stable counting sort, done separately on the two parts of the columns:
// part 0 = [0, b) (the rows use the same permutation, so row r's positive
// stays column r) and part 1 = [b, nc) (the shared negatives). The key of
// column j is bin(id_j), the top 8 bits of the id's Fibonacci hash (as in
// k5_hash); equal ids share a bin, so the columns that can be
// hits of row r lie in the column ranges of bin(r) in both parts. Stable
// ranks make the order, and with it every sum, the same on every run.
//
// Part p is cut into tiles of `tile` elements; hist holds, part after part,
// bin-major, the count of each (bin, tile); its exclusive prefix is the
// sorted position of the first element of each (bin, tile).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int k5_bin(long long id) {
    return (int)(((unsigned long long)id * 0x9E3779B97F4A7C15ull) >> 56);
}

struct SortShape {
    int b, nc, tile, tiles0, tiles1;
    __device__ __forceinline__ void block_part(int blk, int* part, int* t, int* lo, int* hi) const {
        *part = blk < tiles0 ? 0 : 1;
        *t = *part == 0 ? blk : blk - tiles0;
        const int base = *part == 0 ? 0 : b;
        const int end = *part == 0 ? b : nc;
        *lo = base + *t * tile;
        *hi = *lo + tile < end ? *lo + tile : end;
    }
    __device__ __forceinline__ int64_t hist_at(int part, int bin, int t) const {
        return part == 0 ? (int64_t)bin * tiles0 + t : (int64_t)K5_BINS * tiles0 + (int64_t)bin * tiles1 + t;
    }
};

__global__ void __launch_bounds__(K5_SORT_THREADS)
    k5_sort_count(const int64_t* __restrict__ item_ids, SortShape sh, int* __restrict__ hist) {
    __shared__ int h[K5_BINS];
    int part, t, lo, hi;
    sh.block_part(blockIdx.x, &part, &t, &lo, &hi);
    h[threadIdx.x] = 0;
    __syncthreads();
    for (int j = lo + threadIdx.x; j < hi; j += K5_SORT_THREADS) atomicAdd(&h[k5_bin(item_ids[j])], 1);
    __syncthreads();
    hist[sh.hist_at(part, threadIdx.x, t)] = h[threadIdx.x];
}

// One block: exclusive prefix of hist in place, then the bin starts. hist
// has a multiple of 256 entries; each thread scans a slice of whole int4s.
__global__ void __launch_bounds__(K5_SCAN_THREADS)
    k5_sort_scan(SortShape sh, int* __restrict__ hist, int* __restrict__ bstart) {
    __shared__ int warp_tot[K5_SCAN_THREADS / 32];
    const int64_t len4 = (int64_t)K5_BINS / 4 * (sh.tiles0 + sh.tiles1);
    const int64_t per4 = (len4 + K5_SCAN_THREADS - 1) / K5_SCAN_THREADS;
    const int64_t a = threadIdx.x * per4;
    const int64_t e = a + per4 < len4 ? a + per4 : len4;
    int4* h4 = reinterpret_cast<int4*>(hist);
    int mine = 0;
#pragma unroll 4
    for (int64_t q = a; q < e; ++q) {
        const int4 v = h4[q];
        mine += v.x + v.y + v.z + v.w;
    }
    // block exclusive scan of the per-thread totals
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = mine;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive
    }
    __syncthreads();
    int run = inc - mine + (warp > 0 ? warp_tot[warp - 1] : 0);
#pragma unroll 4
    for (int64_t q = a; q < e; ++q) {
        const int4 v = h4[q];
        int4 o;
        o.x = run;
        o.y = o.x + v.x;
        o.z = o.y + v.y;
        o.w = o.z + v.z;
        run = o.w + v.w;
        h4[q] = o;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < 2 * (K5_BINS + 1); k += K5_SCAN_THREADS) {
        const int part = k / (K5_BINS + 1), bin = k % (K5_BINS + 1);
        const int tiles = part == 0 ? sh.tiles0 : sh.tiles1;
        const int end = part == 0 ? sh.b : sh.nc;
        bstart[k] = (bin < K5_BINS && tiles > 0) ? hist[sh.hist_at(part, bin, 0)] : end;
    }
}

// Element j of a tile goes to hist[(bin, tile)] + (elements of its bin
// before it in the tile); the tile is walked in rounds of 256 in index order.
__global__ void __launch_bounds__(K5_SORT_THREADS)
    k5_sort_scatter(const int64_t* __restrict__ item_ids, SortShape sh, const int* __restrict__ hist,
                    int* __restrict__ perm, uint8_t* __restrict__ sbin) {
    __shared__ int run[K5_BINS];
    __shared__ int wcnt[K5_SORT_WARPS][K5_BINS];
    int part, t, lo, hi;
    sh.block_part(blockIdx.x, &part, &t, &lo, &hi);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    run[threadIdx.x] = 0;
    for (int w = 0; w < K5_SORT_WARPS; ++w) wcnt[w][threadIdx.x] = 0;
    __syncthreads();
    for (int r0 = lo; r0 < hi; r0 += K5_SORT_THREADS) {
        const int j = r0 + threadIdx.x;
        const bool in = j < hi;
        const int bin = in ? k5_bin(item_ids[j]) : K5_BINS;  // K5_BINS: no element
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        const int lrank = __popc(peers & ((1u << lane) - 1u));
        if (in && lrank == 0) wcnt[warp][bin] = __popc(peers);
        __syncthreads();
        if (in) {
            int pos = hist[sh.hist_at(part, bin, t)] + run[bin] + lrank;
            for (int w = 0; w < warp; ++w) pos += wcnt[w][bin];
            perm[pos] = j;
            if (part == 0) sbin[pos] = (uint8_t)bin;
        }
        __syncthreads();
        int add = 0;
        for (int w = 0; w < K5_SORT_WARPS; ++w) {
            add += wcnt[w][threadIdx.x];
            wcnt[w][threadIdx.x] = 0;
        }
        run[threadIdx.x] += add;
        __syncthreads();
    }
}

// Sorted position q takes original row perm[q]: items (and, for q < b,
// users) in 16-byte pieces, and the column data.
__global__ void k5_permute(const int* __restrict__ perm, int b, int nc, int vpr, const uint4* __restrict__ users,
                           const uint4* __restrict__ items, const ColInfo* __restrict__ col, uint4* __restrict__ users_s,
                           uint4* __restrict__ items_s, ColInfo* __restrict__ col_s, int* err) {
    const int64_t total = (int64_t)nc * vpr;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total; v += (int64_t)gridDim.x * blockDim.x) {
        const int q = (int)(v / vpr);
        const int piece = (int)(v - (int64_t)q * vpr);
        const int src = perm[q];
        if ((unsigned)src >= (unsigned)(q < b ? b : nc)) {  // never, for a permutation of each part
            atomicExch(err, ERR_BAD_ORDER);
            continue;
        }
        items_s[v] = items[(int64_t)src * vpr + piece];
        if (q < b) users_s[v] = users[(int64_t)src * vpr + piece];
        if (piece == 0) col_s[q] = col[src];
    }
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
    uint8_t* ring = smem + (size_t)p.kchunks * K5_USER_CHUNK;         // [stages][K5_N x 128 B]
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
        // Warp w reads TMEM lanes 32*(w%4).. (its 32 users) and one group of
        // K5_WARP_COLS of the tile's K5_N columns; each thread keeps (max, sum)
        // for its user.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int cgrp = ew >> 2;

        const float2 a2v = make_float2(p.a2, p.a2);
        // TMEM address of chunk c (32 columns) of this warp's slice of accumulator tile tcx
        auto tmem_chunk = [&](uint32_t tcx, int c) -> uint32_t {
            return tmem_base + ((uint32_t)(quarter * 32) << 16) +
                   (uint32_t)((tcx & 1) * K5_ACC_COLS + cgrp * K5_WARP_COLS + c * 32);
        };
        // this warp is done reading accumulator tile tcx
        auto release = [&](uint32_t tcx) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[tcx & 1]);
        };
        uint32_t tc = 0;  // accumulator tiles this CTA has consumed
        bool ok = true;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            int ut, ch, t0, t1;
            unit_cols(p, u, &ut, &ch, &t0, &t1);
            const int i = ut * K5_M + quarter * 32 + lane;  // this thread's user
            const bool row_ok = i < p.b;
            const int my_g = (HITS && row_ok) ? p.col[i].g : -1;
            // Columns where this warp's rows can have hits: the ranges of the
            // bins from its first row's to its last row's, in both parts.
            if constexpr (HITS) {
                __syncwarp();  // the previous unit's reads are done
                if (lane == 0) {
                    int4 r = make_int4(0, 0, 0, 0);
                    const int r0 = ut * K5_M + quarter * 32;
                    if (r0 < p.b) {
                        const int rl = r0 + 31 < p.b ? r0 + 31 : p.b - 1;
                        const int k0 = p.sbin[r0], k1 = p.sbin[rl];
                        r = make_int4(p.bstart[k0], p.bstart[k1 + 1], p.bstart[K5_BINS + 1 + k0],
                                      p.bstart[K5_BINS + 1 + k1 + 1]);
                    }
                    *reinterpret_cast<int4*>(ctl->hit_cols[ew]) = r;
                }
                __syncwarp();
            }
            // Running max m (base-2 units) and sum of 2^(x - m). m is raised
            // only when a chunk's sum leaves [0, 2^64] (terms up to 2^64 are
            // exact enough and far from overflow), so the common path needs
            // no maximum at all.
            float m = K5_MAX_FLOOR;
            float sum = 0.f;

            // One chunk (32 columns) in three parts, so that the next chunk's
            // logits can be formed while this chunk's sum is reduced and tested.
            // Part 1: x = acc * log2(e)/tau + nb_j; the positive's logit; hits
            // (this row's group) set to -inf. Needs no running max.
            auto logits = [&](float* x, int t, int c) {
                const float* nb_s = ctl->nb[ew][t & 1];
                const int* g_s = ctl->grp[ew][t & 1];
                const float4* nb4 = reinterpret_cast<const float4*>(nb_s + c * 32);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 b4 = nb4[e4];
                    const float2 lo = fma2(make_float2(x[4 * e4], x[4 * e4 + 1]), a2v, make_float2(b4.x, b4.y));
                    const float2 hi = fma2(make_float2(x[4 * e4 + 2], x[4 * e4 + 3]), a2v, make_float2(b4.z, b4.w));
                    x[4 * e4] = lo.x;
                    x[4 * e4 + 1] = lo.y;
                    x[4 * e4 + 2] = hi.x;
                    x[4 * e4 + 3] = hi.y;
                }
                const int col0 = t * K5_N + cgrp * K5_WARP_COLS + c * 32;
                if (row_ok && (unsigned)(i - col0) < 32u) {
                    Cols32 tmp;
#pragma unroll
                    for (int e = 0; e < 32; ++e) tmp.x[e] = x[e];
                    p.numer[i] = select32(tmp, i - col0);
                }
                bool maybe_hit = false;
                if constexpr (HITS) {
                    int lo0, hi0, lo1, hi1;
                    asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(lo0), "=r"(hi0), "=r"(lo1), "=r"(hi1)
                                 : "r"(smem_u32(ctl->hit_cols[ew])));
                    maybe_hit = (col0 < hi0 && col0 + 32 > lo0) || (col0 < hi1 && col0 + 32 > lo1);
                }
                if (maybe_hit) {  // warp-uniform
                    const int4* g4 = reinterpret_cast<const int4*>(g_s + c * 32);
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const int4 gg = g4[e4];
                        x[4 * e4] = gg.x == my_g ? -INFINITY : x[4 * e4];
                        x[4 * e4 + 1] = gg.y == my_g ? -INFINITY : x[4 * e4 + 1];
                        x[4 * e4 + 2] = gg.z == my_g ? -INFINITY : x[4 * e4 + 2];
                        x[4 * e4 + 3] = gg.w == my_g ? -INFINITY : x[4 * e4 + 3];
                    }
                }
            };
            // Part 2: the chunk's sum of 2^(x - m).
            auto chunk_sum = [&](const float* x) -> float {
                const float2 nm = make_float2(-m, -m);
                float2 c0 = make_float2(0.f, 0.f), c1 = c0;
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float2 lo = add2(make_float2(x[4 * e4], x[4 * e4 + 1]), nm);
                    float2 hi = add2(make_float2(x[4 * e4 + 2], x[4 * e4 + 3]), nm);
                    lo.x = ex2_approx(lo.x);
                    lo.y = ex2_approx(lo.y);
                    hi.x = ex2_approx(hi.x);
                    hi.y = ex2_approx(hi.y);
                    c0 = add2(c0, lo);
                    c1 = add2(c1, hi);
                }
                const float2 cc = add2(c0, c1);
                return cc.x + cc.y;
            };
            // Part 3: take the sum, or (rare: the running max is too low for this
            // chunk, always on a unit's first chunk) raise the max to the exact
            // chunk max, rescale and sum again.
            auto accumulate = [&](const float* x, float csum) {
                if (csum <= K5_SUM_LIMIT) {
                    sum += csum;
                    return;
                }
                float ca = x[0], cb = x[1];
#pragma unroll
                for (int e = 2; e < 32; e += 4) {
                    ca = max3f(ca, x[e], x[e + 1]);
                    cb = max3f(cb, x[e + 2], x[e + 3]);
                }
                const float cmax = fmaxf(ca, cb);
                if (cmax > m) {
                    sum *= ex2_approx(m - cmax);
                    m = cmax;
                }
                float r0 = 0.f, r1 = 0.f;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    r0 += ex2_approx(x[e] - m);
                    r1 += ex2_approx(x[e + 1] - m);
                }
                sum += r0 + r1;
            };
            // column data of tile t into shared-memory buffer t & 1
            auto stage_cols = [&](int t, const int2* cv) {
                __syncwarp();  // earlier reads of that buffer are done
#pragma unroll
                for (int e = 0; e < K5_WARP_CHUNKS; ++e) {
                    ctl->nb[ew][t & 1][32 * e + lane] = __int_as_float(cv[e].x);
                    ctl->grp[ew][t & 1][32 * e + lane] = cv[e].y;
                }
                __syncwarp();
            };

            // column data: tile t0 into shared memory, t0 + 1 into registers
            int2 ci[K5_WARP_CHUNKS];
#pragma unroll
            for (int e = 0; e < K5_WARP_CHUNKS; ++e) ci[e] = load_col(p, t0 * K5_N + cgrp * K5_WARP_COLS + 32 * e + lane);
            stage_cols(t0, ci);
            if (t0 + 1 < t1) {
#pragma unroll
                for (int e = 0; e < K5_WARP_CHUNKS; ++e)
                    ci[e] = load_col(p, (t0 + 1) * K5_N + cgrp * K5_WARP_COLS + 32 * e + lane);
            }
            // Chunks are loaded from TMEM one ahead of the one being summed,
            // alternating between two register sets (K5_WARP_CHUNKS is even,
            // so chunk c of every tile uses set c & 1).
            Cols32 v[2];
            if (!mbar_wait(&ctl->tfull[tc & 1], (tc >> 1) & 1, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_ld_32cols(tmem_chunk(tc, 0), v[0].x);
            tmem_ld_wait();
            fence_regs(v[0]);
            logits(v[0].x, t0, 0);
            for (int t = t0; t < t1; ++t, ++tc) {
                // column data of tile t + 1 (its first chunk's logits are formed
                // during this tile's last chunk)
                if (t + 1 < t1) {
                    stage_cols(t + 1, ci);
                    if (t + 2 < t1) {
#pragma unroll
                        for (int e = 0; e < K5_WARP_CHUNKS; ++e)
                            ci[e] = load_col(p, (t + 2) * K5_N + cgrp * K5_WARP_COLS + 32 * e + lane);
                    }
                }
#pragma unroll
                for (int c = 0; c < K5_WARP_CHUNKS; ++c) {
                    bool more = true;
                    if (c + 1 < K5_WARP_CHUNKS) {
                        tmem_ld_32cols(tmem_chunk(tc, c + 1), v[(c + 1) & 1].x);
                    } else if (t + 1 < t1) {
                        if (!mbar_wait(&ctl->tfull[(tc + 1) & 1], ((tc + 1) >> 1) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        tmem_ld_32cols(tmem_chunk(tc + 1, 0), v[0].x);
                    } else {
                        more = false;
                    }
                    const float csum = chunk_sum(v[c & 1].x);
                    if (more) {
                        tmem_ld_wait();
                        fence_regs(v[(c + 1) & 1]);
                        if (c + 1 == K5_WARP_CHUNKS - 1) release(tc);  // tile tc fully loaded
                        if (c + 1 < K5_WARP_CHUNKS)
                            logits(v[(c + 1) & 1].x, t, c + 1);
                        else
                            logits(v[0].x, t + 1, 0);
                    }
                    accumulate(v[c & 1].x, csum);
                }
                if (!ok) break;
            }
            if (!ok) break;
            if (row_ok) p.part[(int64_t)(ch * K5_COL_GROUPS + cgrp) * p.b + i] = make_float2(m, sum);
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
             const uint8_t* __restrict__ valid, const int* __restrict__ perm, int b, int hits, const int* err,
             float* lse, float* loss, float* mean, double* block_sum, int* block_rows, unsigned* ticket) {
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
        const int o = perm ? perm[i] : i;  // the row's own index
        const bool o_ok = (unsigned)o < (unsigned)b;  // always, k5_permute checked it
        const bool row_valid = o_ok && (valid ? valid[o] != 0 : true);
        float li = row_valid ? (l2 - num) * K5_LN2 : 0.0f;
        float le = l2 * K5_LN2;
        if (failed) li = le = NAN;
        if (o_ok) {
            lse[o] = le;
            loss[o] = li;
        }
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
    if (last) {  // the last block adds the block sums: a fixed-shape tree, the same on every run
        __threadfence();
        double s = 0.0;
        int n = 0;
        for (unsigned blk = threadIdx.x; blk < gridDim.x; blk += K5_MERGE_THREADS) {
            s += ((volatile double*)block_sum)[blk];
            n += ((volatile int*)block_rows)[blk];
        }
        for (int o = 16; o > 0; o >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, o);
            n += __shfl_xor_sync(0xffffffffu, n, o);
        }
        if ((threadIdx.x & 31) == 0) {
            red_s[threadIdx.x >> 5] = s;
            red_n[threadIdx.x >> 5] = n;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double tot = 0.0;
            long long rows = 0;
            for (int w = 0; w < K5_MERGE_THREADS / 32; ++w) {
                tot += red_s[w];
                rows += red_n[w];
            }
            *mean = failed ? NAN : (rows > 0 ? (float)(tot / (double)rows) : 0.0f);
        }
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
    pl.tile_cols = K5_N;
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
    // bin order: tiles of a multiple of 1024 elements, at most 1024 tiles per part
    pl.sort_tile = 1024 * (int)(((int64_t)nc + (1 << 20) - 1) >> 20);
    if (pl.sort_tile < 1024) pl.sort_tile = 1024;
    pl.sort_tiles0 = item_ids ? (b + pl.sort_tile - 1) / pl.sort_tile : 0;
    pl.sort_tiles1 = item_ids ? (nc - b + pl.sort_tile - 1) / pl.sort_tile : 0;
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
    pl.off_part = take((size_t)chunks * K5_COL_GROUPS * b * sizeof(float2));
    pl.off_keys = take(item_ids ? ((size_t)1 << pl.log2_slots) * sizeof(unsigned long long) : 0);
    pl.off_block_sum = take((size_t)(pl.merge_blocks > 0 ? pl.merge_blocks : 1) * sizeof(double));
    pl.off_block_rows = take((size_t)(pl.merge_blocks > 0 ? pl.merge_blocks : 1) * sizeof(int));
    const size_t row_bytes = (size_t)d * 2;  // bf16
    pl.off_perm = take(item_ids ? (size_t)nc * sizeof(int) : 0);
    pl.off_sbin = take(item_ids ? (size_t)b : 0);
    pl.off_hist = take(item_ids ? (size_t)K5_BINS * (pl.sort_tiles0 + pl.sort_tiles1) * sizeof(int) : 0);
    pl.off_bstart = take(item_ids ? (size_t)2 * (K5_BINS + 1) * sizeof(int) : 0);
    pl.off_col_s = take(item_ids ? (size_t)nc * sizeof(ColInfo) : 0);
    pl.off_users_s = take(item_ids ? (size_t)b * row_bytes : 0);
    pl.off_items_s = take(item_ids ? (size_t)nc * row_bytes : 0);
    pl.bytes = off;
    return pl;
}

// d >= 64: every TMA box is 64 elements (128 bytes) of K wide.
bool softmax_supported(int d) { return d >= 64 && d <= 512 && softmax_stages(d) >= 2; }

cudaError_t launch_softmax(const SoftmaxPlan& pl, const CUtensorMap& tm_users, const CUtensorMap& tm_items,
                           const void* users, const void* items, int b, int nc, int d, float tau, const float* logq,
                           const int64_t* item_ids, const uint8_t* valid, float* lse, float* loss, float* mean,
                           void* workspace, cudaStream_t s, int sm_count) {
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

    int* perm = nullptr;
    if (hits) {
        SortShape sh;
        sh.b = b;
        sh.nc = nc;
        sh.tile = pl.sort_tile;
        sh.tiles0 = pl.sort_tiles0;
        sh.tiles1 = pl.sort_tiles1;
        perm = reinterpret_cast<int*>(ws + pl.off_perm);
        uint8_t* sbin = ws + pl.off_sbin;
        int* hist = reinterpret_cast<int*>(ws + pl.off_hist);
        int* bstart = reinterpret_cast<int*>(ws + pl.off_bstart);
        ColInfo* col_s = reinterpret_cast<ColInfo*>(ws + pl.off_col_s);
        const int sort_blocks = sh.tiles0 + sh.tiles1;
        note_launch_begin(TT_KIND_SOFTMAX, s);
        k5_sort_count<<<sort_blocks, K5_SORT_THREADS, 0, s>>>(item_ids, sh, hist);
        note_launch_end(TT_KIND_SOFTMAX, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launch_begin(TT_KIND_SOFTMAX, s);
        k5_sort_scan<<<1, K5_SCAN_THREADS, 0, s>>>(sh, hist, bstart);
        note_launch_end(TT_KIND_SOFTMAX, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launch_begin(TT_KIND_SOFTMAX, s);
        k5_sort_scatter<<<sort_blocks, K5_SORT_THREADS, 0, s>>>(item_ids, sh, hist, perm, sbin);
        note_launch_end(TT_KIND_SOFTMAX, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int vpr = d / 8;  // 16-byte pieces of a bf16 row
        const int64_t pieces = (int64_t)nc * vpr;
        const int pblocks = (int)((pieces + 255) / 256 < 8 * sm_count ? (pieces + 255) / 256 : 8 * sm_count);
        note_launch_begin(TT_KIND_SOFTMAX, s);
        k5_permute<<<pblocks, 256, 0, s>>>(perm, b, nc, vpr, static_cast<const uint4*>(users),
                                           static_cast<const uint4*>(items), col,
                                           reinterpret_cast<uint4*>(ws + pl.off_users_s),
                                           reinterpret_cast<uint4*>(ws + pl.off_items_s), col_s, err);
        note_launch_end(TT_KIND_SOFTMAX, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        col = col_s;
    }

    K5Params p;
    p.col = col;
    p.sbin = hits ? ws + pl.off_sbin : nullptr;
    p.bstart = hits ? reinterpret_cast<const int*>(ws + pl.off_bstart) : nullptr;
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
    k5_merge<<<pl.merge_blocks, K5_MERGE_THREADS, 0, s>>>(part, pl.chunks * K5_COL_GROUPS, numer, valid, perm, b,
                                                           hits ? 1 : 0, err, lse, loss, mean, block_sum, block_rows,
                                                           ticket);
    note_launch_end(TT_KIND_SOFTMAX, s);
    return cudaGetLastError();
}

}  // namespace tt
