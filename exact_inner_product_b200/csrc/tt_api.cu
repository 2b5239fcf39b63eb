// tt_api.cu - the C ABI: argument validation, the scan plan, kernel
// orchestration, tensor maps, launch accounting and event timing.
//
// How tt_score_topk stays exact without ever materialising the score matrix:
// each scoring pass keeps, per query, only candidates whose key (score, id)
// beats a threshold key theta, and the final selection checks that the pass
// kept everything it had to. Thresholds are estimated on coarser levels of
// the corpus (every 61st row, every 3721st row, ...): the r-th best key of a
// level, taken with r about 3k/61, predicts a filter that keeps about 3k
// candidates of the next finer level. The deepest level is small enough to
// keep every key (no threshold). A query's final pass is exact when it kept
// at least k keys (so every member of the true top-k beat the threshold) and
// its buffer did not overflow; if either fails - which the estimate makes
// rare but never impossible - the query's list is recomputed by the exact
// fallback scan (k_exact.cu), launched at the end of every search, which has
// no capacity limit. The whole search is enqueued on the caller's stream and
// the call returns without waiting: the host never reads a result.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/tt.h"
#include "tt_device.cuh"
#include "tt_internal.h"

#define TT_VERSION_STRING "tt 0.2.0 (sm_100a)"

struct tt_index {
    const void* rows;
    tt_dtype dtype;
    int64_t n;
    int32_t d;
    const float* inv_norm;
    int device;
    // work memory (device), grown on demand, and the stream it was last used on
    void* scratch;
    size_t scratch_bytes;
    void* io;  // staging of tt_score_topk_host: queries in, results out
    size_t io_bytes;
    cudaStream_t last_stream;
    bool used;
    // status block in host-mapped memory, written by the last kernel of a search
    tt::HostStatus* hstat;
    tt::HostStatus* dstat;  // the same block, as the device addresses it
    int64_t seq;            // calls issued on the handle
    int64_t last_pending;   // seq of the last search whose status block reports it (0: none)
    tt_stats last;
    // the flag block of the last search: its estimate tickets are zero there
    // (cleared by the init kernel, or reset by the estimate that used them)
    int* tickets_zero_at;
};

namespace tt {

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local char g_last_error[256] = {0};

static tt_status cuda_fail(cudaError_t e, const char* what) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? TT_ERR_NO_MEMORY : TT_ERR_CUDA;
}

void set_last_error_message(const char* msg) {
    snprintf(g_last_error, sizeof g_last_error, "%s", msg);
}

#define TT_CUDA(call, what)                          \
    do {                                             \
        cudaError_t _e = (call);                     \
        if (_e != cudaSuccess) return cuda_fail(_e, what); \
    } while (0)

// ---------------------------------------------------------------------------
// launch accounting and event timing
// ---------------------------------------------------------------------------
static std::atomic<int64_t> g_launches{0};
static std::mutex g_prof_mu;
static bool g_prof_on = false;
struct ProfRec {
    int kind;
    cudaEvent_t start, stop;
};
static std::vector<ProfRec> g_prof_recs;
static std::vector<cudaEvent_t> g_event_pool;
static cudaEvent_t g_pending_start = nullptr;

static cudaEvent_t pool_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void note_launch_begin(int kind, cudaStream_t s) {
    (void)kind;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (!g_prof_on) return;
    g_pending_start = pool_event();
    if (g_pending_start) cudaEventRecord(g_pending_start, s);
}

void note_launch_end(int kind, cudaStream_t s) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (!g_prof_on || !g_pending_start) return;
    cudaEvent_t stop = pool_event();
    if (!stop) return;
    cudaEventRecord(stop, s);
    g_prof_recs.push_back({kind, g_pending_start, stop});
    g_pending_start = nullptr;
}

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

static bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return false;
    }
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return false;
    }
    return true;
}

bool bf16_tile_tensor_map(const void* base, int64_t rows, int d, int64_t row_pitch_elems,
                          int box_rows, CUtensorMap* tm) {
    return encode_2d(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)d, (uint64_t)rows,
                     (uint64_t)row_pitch_elems * 2u, 64, (uint32_t)box_rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

// int8 rows: boxes of 128 codes (one 128-byte swizzle row) x box_rows rows.
bool i8_tile_tensor_map(const void* base, int64_t rows, int d, int64_t row_pitch_elems,
                        int box_rows, CUtensorMap* tm) {
    return encode_2d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, (uint64_t)d, (uint64_t)rows,
                     (uint64_t)row_pitch_elems, 128, (uint32_t)box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool tile_tensor_map(int dtype, const void* base, int64_t rows, int d, int64_t row_pitch_elems,
                            int box_rows, CUtensorMap* tm) {
    return dtype == TT_I8 ? i8_tile_tensor_map(base, rows, d, row_pitch_elems, box_rows, tm)
                          : bf16_tile_tensor_map(base, rows, d, row_pitch_elems, box_rows, tm);
}

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static bool valid_dtype(int dt) { return dt == TT_F32 || dt == TT_BF16; }
static bool valid_index_dtype(int dt) { return valid_dtype(dt) || dt == TT_I8; }

static tt_status check_d(int32_t d) {
    if (d <= 0) return TT_ERR_INVALID_ARG;
    if (d % 16 != 0 || d > TT_MAX_D) return TT_ERR_UNSUPPORTED;
    return TT_OK;
}

// The pointer must be device (or managed) memory of the current device.
static tt_status check_device_ptr(const void* p, const char* what) {
    if (p == nullptr) return TT_OK;
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
        return TT_ERR_CUDA;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) {
        snprintf(g_last_error, sizeof g_last_error, "%s is not device memory", what);
        return TT_ERR_INVALID_ARG;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr.device != dev) {
        snprintf(g_last_error, sizeof g_last_error, "%s lives on device %d, current is %d", what,
                 attr.device, dev);
        return TT_ERR_INVALID_ARG;
    }
    return TT_OK;
}

static int sm_count_current() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// ---------------------------------------------------------------------------
// scan plan
// ---------------------------------------------------------------------------
// Level i samples every 61^i-th row. A prime stride keeps the samples spread
// over masks that repeat with a period of 2, 4, 8, ... rows (with a stride
// of 64, every sample of `type = id % 4` would have the same type).
constexpr int STRIDE_RATIO = 61;
constexpr int DEFAULT_CAP = 16384;
constexpr int MAX_DEEPEST_ROWS = 4096;  // the deepest level keeps every key
// Floors of the ranks. The survivors of a pass whose threshold is the r-th
// best key of a 1/61 sample number about Gamma(r, 61); a pass that must keep
// `need` keys falls short with probability P(Poisson(need / 61) >= r).
// Level 1 sets the threshold of the full pass (need = k): r >= max(3k/61, 32)
// puts that below 1e-8 per query. Deeper levels only feed a coarser pass
// (need <= a few dozen, so need / 61 < 1) and 10 suffices there, with far
// fewer keys kept per pass.
constexpr int MIN_RANK = 32;
constexpr int MIN_RANK_DEEP = 10;
// Batches at least this large, on a corpus stored normalised, go to the
// tensor-core kernel on SM pairs (queries in tiles of 256 on TMEM lanes);
// the rest to the single-SM kernel (queries in tiles of up to 256 on TMEM
// columns, multiples of 32). Measured on B200 (level-0 pass): 50M x 128
// stored rows, 1024 queries: 13.3 ms on pairs vs 14.6 ms single-SM; 20M x
// 256 raw rows with per-row norms, 4096 queries: 41.3 ms vs 36.4 ms, so
// corpora with per-row norms stay on the single-SM kernel.
constexpr int PAIR_MIN_BATCH = 256;

// P(X >= r) for X ~ Poisson(lambda), r >= 1 (small when lambda < r).
static double poisson_upper(double lambda, int r) {
    if (lambda <= 0.0) return 0.0;
    if (lambda >= r) return 1.0;
    double t = exp(-lambda + r * log(lambda) - lgamma(r + 1.0)), sum = 0.0;
    for (int i = r; i < r + 2000 && t > sum * 1e-17; ++i) {
        sum += t;
        t *= lambda / (i + 1);
    }
    return sum;
}

// P(X < r) for X ~ Poisson(mu).
static double poisson_lower(double mu, int r) {
    double sum = 0.0;
    for (int i = 0; i < r; ++i) sum += exp(-mu + i * log(mu) - lgamma(i + 1.0));
    return sum;
}

// The sampled plan of a small batch: one sample of about SAMPLE_ROWS rows
// (every S-th row, S odd, so that masks repeating every 2, 4, 8 ... rows are
// sampled evenly), reduced to the threshold in one launch. The rank r is the
// smallest for which the true top-k misses the filter with probability at
// most PLAN_FAIL_P (more than r - 1 sample rows among the true top k - 1, a
// Poisson(k / S) count), and the filter must also keep at most `cap` rows with
// that probability (fewer than r sample rows among the best cap, a
// Poisson(cap / S) count). Returns false when no such plan exists.
constexpr int64_t SAMPLE_ROWS = 16384;
constexpr double PLAN_FAIL_P = 1e-9;

static bool sampled_plan(int64_t n, int32_t k, int cap, int scale, Plan* p) {
    if (n <= 2 * SAMPLE_ROWS) return false;
    int64_t S = n / SAMPLE_ROWS;
    if ((S & 1) == 0) ++S;
    const int64_t ns = (n + S - 1) / S;
    const double f = (double)ns / (double)n;
    int r = 1;
    while (r <= 256 && poisson_upper(k * f, r) > PLAN_FAIL_P) ++r;
    if (r > 256 || poisson_lower(cap * f, r) > PLAN_FAIL_P) return false;
    r = (int)((int64_t)r * scale / 100);
    if (r < 1) r = 1;
    if (r > ESTIMATE_MAX_RANK) return false;
    const int64_t blocks = (ns + ESTIMATE_BLOCK_ROWS - 1) / ESTIMATE_BLOCK_ROWS;
    if (blocks * r > 4096 || blocks * r > cap) return false;  // the blocks' lists are merged in shared memory
    p->levels = 2;
    p->sampled = true;
    p->stride[0] = 1;
    p->rows[0] = n;
    p->rank[0] = k;
    p->stride[1] = S;
    p->rows[1] = ns;
    p->rank[1] = r;
    return true;
}

tt_status make_plan(int64_t n, int32_t k, const tt_options* opt, bool small_batch, Plan* p) {
    int cap = (opt && opt->cap) ? opt->cap : DEFAULT_CAP;
    if (cap < 256 || cap > DEFAULT_CAP || (cap & (cap - 1)) != 0) return TT_ERR_INVALID_ARG;
    if (cap < 2 * k) return TT_ERR_INVALID_ARG;
    const int scale = (opt && opt->rank_scale_pct) ? opt->rank_scale_pct : 100;
    if (scale < 1 || scale > 10000) return TT_ERR_INVALID_ARG;
    const int forced = opt ? opt->force_levels : 0;
    if (forced < 0 || forced > MAX_LEVELS) return TT_ERR_INVALID_ARG;
    p->cap = cap;
    p->sampled = false;
    if (small_batch && forced == 0 && sampled_plan(n, k, cap, scale, p)) return TT_OK;
    int L = 0;
    int64_t s = 1;
    if (forced > 0) {
        L = forced - 1;
        for (int i = 0; i < L; ++i) s *= STRIDE_RATIO;
        while (L > 0 && s >= n) {  // keep at least two rows at the deepest level
            s /= STRIDE_RATIO;
            --L;
        }
    } else {
        const int64_t deepest = cap < MAX_DEEPEST_ROWS ? cap : MAX_DEEPEST_ROWS;
        while ((n + s - 1) / s > deepest && L < MAX_LEVELS - 1) {
            s *= STRIDE_RATIO;
            ++L;
        }
    }
    p->levels = L + 1;
    int64_t st = 1;
    int need = k;  // rank needed at the finer level
    p->rank[0] = k;
    for (int i = 0; i <= L; ++i) {
        p->stride[i] = st;
        p->rows[i] = n > 0 ? (n + st - 1) / st : 0;
        if (i >= 1) {
            int64_t r = (3 * (int64_t)need + STRIDE_RATIO - 1) / STRIDE_RATIO;
            const int floor_r = i == 1 ? MIN_RANK : MIN_RANK_DEEP;
            if (r < floor_r) r = floor_r;
            r = r * scale / 100;
            if (r < 1) r = 1;
            p->rank[i] = (int)r;
            need = (int)r;
        }
        st *= STRIDE_RATIO;
    }
    return TT_OK;
}

// ---------------------------------------------------------------------------
// scratch
// ---------------------------------------------------------------------------
struct Scratch {
    uint64_t* keys;
    uint32_t* count;
    uint64_t* theta;
    float* thf;
    int32_t* flagged;  // lists handed to the exact fallback
    int* flags;        // [0] flagged lists, [1] error word of expired device waits
    __nv_bfloat16* qcast;
    int8_t* qcodes;   // int8 index: the queries' codes [b, d]
    float* qscale;    // and their scales [b]
    // several result sets by type: per-query minima of the virtual
    // thresholds [b_pad] and the type -> set map [256]
    uint64_t* theta_min;
    float* thf_min;
    int8_t* set_of;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Work blocks released by a handle (tt_free, or growth) are kept here, per
// device, and handed to later handles, so that short-lived handles do not
// cudaMalloc/cudaFree on every call (cudaFree waits for the whole device).
// Work still queued on the stream that last used a block may read it, so a
// block carries an event recorded on that stream, and a later user's stream
// waits for it before any of its own work touches the block. Blocks stay with
// the process until it exits.
struct PooledBlock {
    int device;
    void* ptr;
    size_t bytes;
    cudaEvent_t ready;  // null: nothing queued used it
};
static std::mutex g_pool_mu;
static std::vector<PooledBlock> g_pool;

static void* pool_take(int device, size_t need, size_t* got, cudaStream_t s) {
    PooledBlock blk{};
    {
        std::lock_guard<std::mutex> lock(g_pool_mu);
        int best = -1;
        for (int i = 0; i < (int)g_pool.size(); ++i)
            if (g_pool[i].device == device && g_pool[i].bytes >= need &&
                (best < 0 || g_pool[i].bytes < g_pool[best].bytes))
                best = i;
        if (best < 0) return nullptr;
        blk = g_pool[best];
        g_pool.erase(g_pool.begin() + best);
    }
    if (blk.ready) {
        cudaStreamWaitEvent(s, blk.ready, 0);
        cudaEventDestroy(blk.ready);
    }
    *got = blk.bytes;
    return blk.ptr;
}

static void pool_give(int device, void* ptr, size_t bytes, cudaStream_t last, bool used) {
    if (!ptr) return;
    cudaEvent_t ev = nullptr;
    if (used && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess) {
        if (cudaEventRecord(ev, last) != cudaSuccess) {
            cudaGetLastError();
            cudaEventDestroy(ev);
            ev = nullptr;
            cudaStreamSynchronize(last);  // no event: make sure nothing queued still reads the block
            cudaGetLastError();
        }
    }
    std::lock_guard<std::mutex> lock(g_pool_mu);
    g_pool.push_back({device, ptr, bytes, ev});
}

// A block of at least `need` bytes for *slot (a handle's scratch or io),
// replacing the current one when it is too small.
static tt_status grow_block(tt_index* ix, void** slot, size_t* slot_bytes, size_t need, cudaStream_t s,
                            const char* what) {
    if (need <= *slot_bytes) return TT_OK;
    if (*slot) {
        pool_give(ix->device, *slot, *slot_bytes, ix->last_stream, ix->used);
        *slot = nullptr;
        *slot_bytes = 0;
    }
    size_t got = 0;
    void* p = pool_take(ix->device, need, &got, s);
    if (!p) {
        got = need + need / 4;
        cudaError_t e = cudaMalloc(&p, got);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, what);
        }
    }
    *slot = p;
    *slot_bytes = got;
    return TT_OK;
}

// Status blocks (host-mapped, one per handle), reused the same way; a block
// is handed out again only once the work that may still write it is done.
struct PooledStatus {
    HostStatus* p;
    cudaEvent_t done;  // null: nothing queued writes it
};
static std::vector<PooledStatus> g_status_pool;

static HostStatus* status_take() {
    {
        std::lock_guard<std::mutex> lock(g_pool_mu);
        for (size_t i = 0; i < g_status_pool.size(); ++i) {
            PooledStatus ps = g_status_pool[i];
            if (ps.done) {
                if (cudaEventQuery(ps.done) != cudaSuccess) {
                    cudaGetLastError();
                    continue;
                }
                cudaEventDestroy(ps.done);
            }
            g_status_pool.erase(g_status_pool.begin() + (long)i);
            return ps.p;
        }
    }
    void* p = nullptr;
    if (cudaHostAlloc(&p, 64, cudaHostAllocMapped) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return static_cast<HostStatus*>(p);
}

static void status_give(HostStatus* p, cudaStream_t last = nullptr, bool used = false) {
    if (!p) return;
    cudaEvent_t ev = nullptr;
    if (used && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(ev, last) != cudaSuccess) {
        cudaGetLastError();
        cudaEventDestroy(ev);
        ev = nullptr;
        cudaStreamSynchronize(last);
        cudaGetLastError();
    }
    std::lock_guard<std::mutex> lock(g_pool_mu);
    g_status_pool.push_back({p, ev});
}

// A device wait of an earlier search on this handle expired (its outputs were
// set to id -1, score NaN): report it once, as TT_ERR_TIMEOUT.
static tt_status report_pending(tt_index* ix) {
    if (ix->hstat && ix->hstat->err != 0) {
        const int code = ix->hstat->err;
        ix->hstat->err = 0;
        snprintf(g_last_error, sizeof g_last_error,
                 "a device-side wait expired in a search on this handle (code %d); that search's outputs "
                 "hold id -1 and score NaN", code);
        return TT_ERR_TIMEOUT;
    }
    return TT_OK;
}

// b, b_pad: queries (with the padding of the query tiles); vq, vpad: the
// lists kept (vq = b, or sets * b for several result sets, padded to vpad);
// n_min: entries of the per-query minima (0 without result sets).
static tt_status get_scratch(tt_index* ix, int b, int b_pad, int vq, int vpad, int n_min, int cap, int d,
                             bool need_qcast, bool need_q8, cudaStream_t s, Scratch* out) {
    size_t off = 0;
    const size_t o_keys = off;
    off = align_up(off + (size_t)vq * cap * 8, 256);
    const size_t o_count = off;
    off = align_up(off + (size_t)vpad * 4, 256);
    const size_t o_theta = off;
    off = align_up(off + (size_t)vpad * 8, 256);
    const size_t o_thf = off;
    off = align_up(off + (size_t)vpad * 4, 256);
    const size_t o_flagged = off;
    off = align_up(off + (size_t)vpad * 4, 256);
    const size_t o_tmin = off;
    off = align_up(off + (size_t)n_min * 8, 256);
    const size_t o_fmin = off;
    off = align_up(off + (size_t)n_min * 4, 256);
    const size_t o_setof = off;
    off = align_up(off + (n_min > 0 ? 256 : 0), 256);
    const size_t o_flags = off;
    off = align_up(off + 64, 256);
    const size_t o_q = off;
    off = align_up(off + (need_qcast ? (size_t)b * d * 2 : 0), 256);
    const size_t o_q8 = off;
    off = align_up(off + (need_q8 ? (size_t)b * d : 0), 256);
    const size_t o_qs = off;
    off = align_up(off + (need_q8 ? (size_t)b_pad * 4 : 0), 256);
    tt_status st = grow_block(ix, &ix->scratch, &ix->scratch_bytes, off, s, "scratch allocation");
    if (st != TT_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(ix->scratch);
    out->keys = reinterpret_cast<uint64_t*>(base + o_keys);
    out->count = reinterpret_cast<uint32_t*>(base + o_count);
    out->theta = reinterpret_cast<uint64_t*>(base + o_theta);
    out->thf = reinterpret_cast<float*>(base + o_thf);
    out->flagged = reinterpret_cast<int32_t*>(base + o_flagged);
    out->flags = reinterpret_cast<int*>(base + o_flags);
    out->qcast = need_qcast ? reinterpret_cast<__nv_bfloat16*>(base + o_q) : nullptr;
    out->qcodes = need_q8 ? reinterpret_cast<int8_t*>(base + o_q8) : nullptr;
    out->qscale = need_q8 ? reinterpret_cast<float*>(base + o_qs) : nullptr;
    out->theta_min = n_min > 0 ? reinterpret_cast<uint64_t*>(base + o_tmin) : nullptr;
    out->thf_min = n_min > 0 ? reinterpret_cast<float*>(base + o_fmin) : nullptr;
    out->set_of = n_min > 0 ? reinterpret_cast<int8_t*>(base + o_setof) : nullptr;
    if (!ix->hstat) {
        ix->hstat = status_take();
        void* dp = nullptr;
        if (!ix->hstat || cudaHostGetDevicePointer(&dp, (void*)ix->hstat, 0) != cudaSuccess) {
            cudaGetLastError();
            status_give(ix->hstat);
            ix->hstat = nullptr;
            snprintf(g_last_error, sizeof g_last_error, "mapped status block allocation failed");
            return TT_ERR_NO_MEMORY;
        }
        ix->dstat = static_cast<HostStatus*>(dp);
        ix->hstat->err = 0;
        ix->hstat->seq_repaired = 0;
    }
    return TT_OK;
}

// ---------------------------------------------------------------------------
// one scoring pass over level i
// ---------------------------------------------------------------------------
struct PathCfg {
    int path;           // 1 stream, 2 tensor, 3 tensor on SM pairs
    int nq;             // tensor path: queries per tile
    const void* queries;
    int q_dtype;
    const float* qscale;  // int8 index: query scales
    int withhold_copy;    // test hook, see tt_options
    const uint8_t* types; // several result sets by type: the candidates' types, else null
    CUtensorMap tm_q;
};

static tt_status run_pass(const tt_index* ix, const PathCfg& pc, const Plan& plan, int level,
                          const Scratch& sc, const uint32_t* exclude, float inv_tau, int b,
                          cudaStream_t s, int sms) {
    PassArgs a;
    a.rows = ix->rows;
    a.dtype = ix->dtype;
    a.n_rows = plan.rows[level];
    a.stride = plan.stride[level];
    a.d = ix->d;
    a.inv_norm = ix->inv_norm;
    a.exclude = exclude;
    a.inv_tau = inv_tau;
    a.queries = pc.queries;
    a.q_dtype = pc.q_dtype;
    a.qscale = pc.qscale;
    a.withhold_copy = pc.withhold_copy;
    a.b = b;
    a.theta = sc.theta;
    a.thf = sc.thf;
    a.count = sc.count;
    a.keys = sc.keys;
    a.cap = plan.cap;
    a.err = sc.flags + 1;
    a.types = pc.types;
    a.set_of = pc.types ? sc.set_of : nullptr;
    a.defer = (plan.sampled && level == 0) ? 1 : 0;  // the pass right after the one-sample estimate
    a.theta_v = pc.types ? sc.theta : nullptr;
    if (pc.types) {  // first tests against each query's loosest set threshold
        a.theta = sc.theta_min;
        a.thf = sc.thf_min;
    }
    cudaError_t e;
    if (pc.path == 2) {
        CUtensorMap tm_rows;
        if (!tile_tensor_map(ix->dtype, ix->rows, a.n_rows, ix->d, a.stride * ix->d, 128, &tm_rows))
            return TT_ERR_CUDA;
        e = launch_tensor_pass(a, tm_rows, pc.tm_q, pc.nq, s, sms);
    } else if (pc.path == 3) {
        CUtensorMap tm_rows;
        if (!tile_tensor_map(ix->dtype, ix->rows, a.n_rows, ix->d, a.stride * ix->d, tensor_pair_box_rows(ix->d),
                             &tm_rows))
            return TT_ERR_CUDA;
        e = launch_tensor_pair_pass(a, tm_rows, s, sms);
    } else {
        e = launch_stream_pass(a, s, sms);
    }
    if (e != cudaSuccess) return cuda_fail(e, pc.path == 1 ? "stream pass" : "tensor pass");
    return TT_OK;
}

}  // namespace tt

using namespace tt;

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* tt_version(void) { return TT_VERSION_STRING; }

const char* tt_status_string(tt_status st) {
    switch (st) {
        case TT_OK: return "TT_OK";
        case TT_ERR_INVALID_ARG: return "TT_ERR_INVALID_ARG";
        case TT_ERR_UNSUPPORTED: return "TT_ERR_UNSUPPORTED";
        case TT_ERR_CUDA: return "TT_ERR_CUDA";
        case TT_ERR_NO_MEMORY: return "TT_ERR_NO_MEMORY";
        case TT_ERR_TIMEOUT: return "TT_ERR_TIMEOUT";
        case TT_ERR_INTERNAL: return "TT_ERR_INTERNAL";
    }
    return "TT_ERR_UNKNOWN";
}

const char* tt_last_error(void) { return g_last_error; }

int64_t tt_launch_count(void) { return g_launches.load(); }

tt_status tt_profile_begin(void) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    for (auto& r : g_prof_recs) {
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_prof_recs.clear();
    g_prof_on = true;
    return TT_OK;
}

tt_status tt_profile_launches(int32_t* kinds, double* ms, int32_t max_records, int32_t* n_records) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    int32_t n = 0;
    for (auto& r : g_prof_recs) {
        if (n >= max_records) break;
        float t = 0.f;
        cudaError_t e = cudaEventSynchronize(r.stop);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.stop);
        if (e != cudaSuccess) return cuda_fail(e, "profile event");
        if (kinds) kinds[n] = r.kind;
        if (ms) ms[n] = t;
        ++n;
    }
    if (n_records) *n_records = n;
    return TT_OK;
}

tt_status tt_profile_end(double* ms_per_kind, int64_t* launches_per_kind) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_prof_on = false;
    double ms[TT_NUM_KINDS] = {0};
    int64_t cnt[TT_NUM_KINDS] = {0};
    tt_status st = TT_OK;
    for (auto& r : g_prof_recs) {
        float t = 0.f;
        cudaError_t e = cudaEventSynchronize(r.stop);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.stop);
        if (e != cudaSuccess) {
            st = cuda_fail(e, "profile event");
            continue;
        }
        if (r.kind >= 0 && r.kind < TT_NUM_KINDS) {
            ms[r.kind] += t;
            cnt[r.kind] += 1;
        }
    }
    for (auto& r : g_prof_recs) {
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_prof_recs.clear();
    for (int i = 0; i < TT_NUM_KINDS; ++i) {
        if (ms_per_kind) ms_per_kind[i] = ms[i];
        if (launches_per_kind) launches_per_kind[i] = cnt[i];
    }
    return st;
}

tt_status tt_plan(int64_t n, int32_t k, const tt_options* options, int32_t* levels,
                  int64_t* rows, int64_t* strides, int32_t* ranks, int32_t* cap) {
    if (n < 0 || n > TT_MAX_N) return TT_ERR_INVALID_ARG;
    if (k <= 0) return TT_ERR_INVALID_ARG;
    if (k > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    Plan p;
    tt_status st = make_plan(n, k, options, false, &p);
    if (st != TT_OK) return st;
    if (levels) *levels = p.levels;
    if (cap) *cap = p.cap;
    for (int i = 0; i < p.levels; ++i) {
        if (rows) rows[i] = p.rows[i];
        if (strides) strides[i] = p.stride[i];
        if (ranks) ranks[i] = p.rank[i];
    }
    return TT_OK;
}

static tt_status new_index(const void* rows, tt_dtype dtype, int64_t n, int32_t d,
                           const float* inv_norm, tt_index** index_out) {
    tt_index* ix = new (std::nothrow) tt_index;
    if (!ix) return TT_ERR_NO_MEMORY;
    memset(ix, 0, sizeof *ix);
    ix->rows = rows;
    ix->dtype = dtype;
    ix->n = n;
    ix->d = d;
    ix->inv_norm = inv_norm;
    cudaGetDevice(&ix->device);
    *index_out = ix;
    return TT_OK;
}

tt_status tt_normalize_candidates(const void* in, tt_dtype in_dtype, int64_t n, int32_t d,
                                  void* out, tt_dtype out_dtype, int32_t mode, void* stream,
                                  tt_index** index_out) {
    // host-side checks first: nothing touches the device before they pass
    if (index_out) *index_out = nullptr;
    if (n < 0) return TT_ERR_INVALID_ARG;
    if (n > TT_MAX_N) return TT_ERR_UNSUPPORTED;
    tt_status st = check_d(d);
    if (st != TT_OK) return st;
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return TT_ERR_INVALID_ARG;
    if (mode != TT_NORM_STORE && mode != TT_NORM_FUSED) return TT_ERR_INVALID_ARG;
    if (n > 0 && (in == nullptr || out == nullptr)) return TT_ERR_INVALID_ARG;
    if (!aligned(in, 16) || !aligned(out, 16)) return TT_ERR_INVALID_ARG;
    if (n > 0) {
        if ((st = check_device_ptr(in, "in")) != TT_OK) return st;
        if ((st = check_device_ptr(out, "out")) != TT_OK) return st;
        cudaError_t e = launch_normalize(in, in_dtype, n, d, out, out_dtype, mode,
                                         static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "normalize");
    }
    if (index_out) {
        if (mode == TT_NORM_STORE)
            return new_index(out, out_dtype, n, d, nullptr, index_out);
        return new_index(in, in_dtype, n, d, static_cast<const float*>(out), index_out);
    }
    return TT_OK;
}

tt_status tt_quantize_candidates(const void* in, tt_dtype in_dtype, int64_t n, int32_t d, int8_t* out_codes,
                                 float* out_scales, void* stream, tt_index** index_out) {
    if (index_out) *index_out = nullptr;
    if (n < 0) return TT_ERR_INVALID_ARG;
    if (n > TT_MAX_N) return TT_ERR_UNSUPPORTED;
    tt_status st = check_d(d);
    if (st != TT_OK) return st;
    if (!valid_dtype(in_dtype)) return TT_ERR_INVALID_ARG;
    if (n > 0 && (in == nullptr || out_codes == nullptr || out_scales == nullptr)) return TT_ERR_INVALID_ARG;
    if (!aligned(in, 16) || !aligned(out_codes, 16) || !aligned(out_scales, 4)) return TT_ERR_INVALID_ARG;
    if (n > 0) {
        if ((st = check_device_ptr(in, "in")) != TT_OK) return st;
        if ((st = check_device_ptr(out_codes, "out_codes")) != TT_OK) return st;
        if ((st = check_device_ptr(out_scales, "out_scales")) != TT_OK) return st;
        cudaError_t e = launch_quantize(in, in_dtype, n, d, out_codes, out_scales, true,
                                        static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "quantize");
    }
    if (index_out) return new_index(out_codes, TT_I8, n, d, out_scales, index_out);
    return TT_OK;
}

tt_status tt_index_wrap(const void* rows, tt_dtype dtype, int64_t n, int32_t d,
                        const float* inv_norm, tt_index** index_out) {
    if (!index_out) return TT_ERR_INVALID_ARG;
    *index_out = nullptr;
    if (n < 0) return TT_ERR_INVALID_ARG;
    if (n > TT_MAX_N) return TT_ERR_UNSUPPORTED;
    tt_status st = check_d(d);
    if (st != TT_OK) return st;
    if (!valid_index_dtype(dtype)) return TT_ERR_INVALID_ARG;
    if (n > 0 && rows == nullptr) return TT_ERR_INVALID_ARG;
    if (dtype == TT_I8 && n > 0 && inv_norm == nullptr) return TT_ERR_INVALID_ARG;  // scales required
    if (!aligned(rows, 16) || !aligned(inv_norm, 4)) return TT_ERR_INVALID_ARG;
    if (n > 0) {
        if ((st = check_device_ptr(rows, "rows")) != TT_OK) return st;
        if ((st = check_device_ptr(inv_norm, "inv_norm")) != TT_OK) return st;
    }
    return new_index(rows, dtype, n, d, inv_norm, index_out);
}

void tt_free(tt_index* index) {
    if (!index) return;
    pool_give(index->device, index->scratch, index->scratch_bytes, index->last_stream, index->used);
    pool_give(index->device, index->io, index->io_bytes, index->last_stream, index->used);
    status_give(index->hstat, index->last_stream, index->used);
    delete index;
}

tt_status tt_last_stats(const tt_index* index, tt_stats* out) {
    if (!index || !out) return TT_ERR_INVALID_ARG;
    *out = index->last;
    if (index->last_pending != 0 && index->hstat) {  // known once the call's last kernel has run
        const uint64_t w = index->hstat->seq_repaired;
        out->rescans = (uint32_t)(w >> 32) == (uint32_t)index->last_pending ? (int32_t)(uint32_t)w : -1;
    } else if (index->last_pending != 0) {
        out->rescans = -1;
    }
    return TT_OK;
}

tt_status tt_index_check(tt_index* index, void* stream) {
    if (!index) return TT_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    return report_pending(index);
}

// The whole search. With `types`, one pass serves n_sets result sets: set t
// takes the candidates whose type maps to t (set_of_host, 256 entries, -1 for
// none), and its lists are out_ids[t * b * k ...] (virtual queries t * b + q).
static tt_status score_core(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                            const uint32_t* exclude_bits, float tau, int32_t k, int32_t* out_ids,
                            float* out_scores, void* stream, const tt_options* options, const uint8_t* types,
                            int n_sets, const int8_t* set_of_host) {
    // ---------------- host-side validation (no device calls) ----------------
    if (!index) return TT_ERR_INVALID_ARG;
    if (b < 0) return TT_ERR_INVALID_ARG;
    if (k <= 0) return TT_ERR_INVALID_ARG;
    if (k > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    if (!(tau > 0.0f) || !isfinite(tau)) return TT_ERR_INVALID_ARG;
    if (!valid_dtype(q_dtype)) return TT_ERR_INVALID_ARG;
    if (b > 0 && (queries == nullptr || out_ids == nullptr || out_scores == nullptr))
        return TT_ERR_INVALID_ARG;
    if (!aligned(queries, 16) || !aligned(out_ids, 4) || !aligned(out_scores, 4) ||
        !aligned(exclude_bits, 4))
        return TT_ERR_INVALID_ARG;
    const int path_req = options ? options->path : 0;
    if (path_req < 0 || path_req > 3) return TT_ERR_INVALID_ARG;
    tt_status st;
    if (index->dtype == TT_F32 && index->d > 256) return TT_ERR_UNSUPPORTED;
    const bool i8 = index->dtype == TT_I8;
    // int8 rows are read in 32-byte pieces by the streaming scorer
    if (i8 && index->d % 32 != 0) return TT_ERR_UNSUPPORTED;
    const int esize = i8 ? 1 : 2;
    const bool tc_possible = (index->dtype == TT_BF16 || i8) && index->d >= 64 &&
                             tensor_pass_max_nq(index->d, esize) > 0;
    // SM pairs: bf16 rows, or int8 codes (not with several result sets)
    const bool pair_possible = (index->dtype == TT_BF16 || (i8 && types == nullptr)) && index->d >= 64 &&
                               tensor_pair_smem_bytes(index->d, esize) > 0;
    int path = path_req;
    if (path == 0) {
        path = 1;
        if (tc_possible && b > 8) path = 2;
        // rows with norms stay on the single-SM kernel (measured faster there);
        // int8 scales take the pair kernel's integer fast test
        if (pair_possible && b >= PAIR_MIN_BATCH && (index->inv_norm == nullptr || i8)) path = 3;
    }
    if (path == 2 && !tc_possible) return TT_ERR_UNSUPPORTED;
    if (path == 3 && !pair_possible) return TT_ERR_UNSUPPORTED;
    // a few queries on the streaming scorer: one sample sets the threshold
    Plan plan;
    if ((st = make_plan(index->n, k, options, path == 1 && types == nullptr && b <= 8, &plan)) != TT_OK) return st;
    if (b == 0) return TT_OK;
    const int V = types ? n_sets * b : b;  // lists kept: one per (set, query)

    // ---------------- device checks ----------------
    if ((st = check_device_ptr(queries, "queries")) != TT_OK) return st;
    if ((st = check_device_ptr(out_ids, "out_ids")) != TT_OK) return st;
    if ((st = check_device_ptr(out_scores, "out_scores")) != TT_OK) return st;
    if ((st = check_device_ptr(exclude_bits, "exclude_bits")) != TT_OK) return st;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != index->device) {
        snprintf(g_last_error, sizeof g_last_error, "index was made on device %d, current is %d",
                 index->device, dev);
        return TT_ERR_INVALID_ARG;
    }
    if ((st = report_pending(index)) != TT_OK) return st;  // an earlier search's expired wait
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t launches0 = g_launches.load();
    tt_stats stats;
    memset(&stats, 0, sizeof stats);
    stats.path = path;
    stats.levels = plan.levels;
    stats.cap = plan.cap;
    stats.sampled = plan.sampled ? 1 : 0;
    for (int i = 0; i < plan.levels; ++i) {
        stats.level_rows[i] = plan.rows[i];
        stats.level_stride[i] = plan.stride[i];
    }

    if (index->n == 0) {
        cudaError_t e = launch_pad(out_ids, out_scores, (int64_t)V * k, s);
        if (e != cudaSuccess) return cuda_fail(e, "pad");
        stats.launches = (int)(g_launches.load() - launches0);
        index->last = stats;
        index->last_pending = 0;
        return TT_OK;
    }

    // Query tiling of the tensor-core path (decided before the scratch layout:
    // threshold arrays are padded to whole query tiles plus one 32-column chunk).
    int nq = 0, q_tiles = 1;
    if (path == 2) {
        const int max_nq = tensor_pass_max_nq(index->d, esize);
        q_tiles = (b + max_nq - 1) / max_nq;
        nq = (b + q_tiles - 1) / q_tiles;
        nq = (nq + 31) / 32 * 32;  // whole 32-column chunks: no chunk reads past the tile
        if (nq > max_nq) nq = max_nq;
    }
    if (path == 3) q_tiles = (b + 255) / 256;
    const int b_pad = (path == 2 ? q_tiles * nq : path == 3 ? q_tiles * 256 : b) + 64;
    const bool need_qcast = !i8 && path >= 2 && q_dtype == TT_F32;
    Scratch sc;
    const int v_pad = types ? V + 64 : b_pad;
    if ((st = get_scratch(index, b, b_pad, V, v_pad, types ? b_pad : 0, plan.cap, index->d, need_qcast, i8, s,
                          &sc)) != TT_OK)
        return st;
    index->last_stream = s;
    index->used = true;
    const int64_t seq = ++index->seq;
    const int sms = sm_count_current();
    const float inv_tau = 1.0f / tau;

    PathCfg pc;
    memset(&pc, 0, sizeof pc);
    pc.path = path;
    pc.queries = queries;
    pc.q_dtype = q_dtype;
    pc.withhold_copy = options ? options->withhold_copy : 0;
    pc.types = types;
    if (types) TT_CUDA(cudaMemcpyAsync(sc.set_of, set_of_host, 256, cudaMemcpyHostToDevice, s), "set map");
    // several result sets: every kernel's first test uses each query's loosest set threshold
    auto sets_min = [&]() -> cudaError_t {
        return types ? launch_sets_min(sc.theta, sc.thf, n_sets, b, b_pad, sc.theta_min, sc.thf_min, s)
                     : cudaSuccess;
    };
    if (i8) {
        // code the queries as given (recsys_two_tower_model.py `compute_top_k_int8`)
        cudaError_t e = launch_quantize(queries, q_dtype, b, index->d, sc.qcodes, sc.qscale, false, s);
        if (e != cudaSuccess) return cuda_fail(e, "query coding");
        pc.queries = sc.qcodes;
        pc.q_dtype = TT_I8;
        pc.qscale = sc.qscale;
    }
    if (path >= 2) {
        if (need_qcast) {
            cudaError_t e = launch_cast_bf16(static_cast<const float*>(queries), (int64_t)b * index->d,
                                             sc.qcast, s);
            if (e != cudaSuccess) return cuda_fail(e, "query cast");
            pc.queries = sc.qcast;
            pc.q_dtype = TT_BF16;
        }
        pc.nq = path == 2 ? nq : 256;
        // single-CTA kernel: the query tile by TMA, boxes of nq queries (the
        // SM-pair kernel reads its queries into tensor memory directly)
        if (path == 2 && !tile_tensor_map(pc.q_dtype, pc.queries, b, index->d, index->d, nq, &pc.tm_q))
            return TT_ERR_CUDA;
    }

    // With one sample the estimate is the first kernel and clears the counters
    // and flags itself, when its tickets are known to be zero: the last search
    // on this handle used the same flag block (the block moves with b and k).
    const bool estimate_clears = plan.sampled && sc.flags == index->tickets_zero_at;
    cudaError_t e = estimate_clears ? cudaSuccess
                                    : launch_init(sc.count, sc.theta, sc.thf, KEY_MIN, V, v_pad, sc.flags, s);
    if (e == cudaSuccess) e = sets_min();
    if (e != cudaSuccess) return cuda_fail(e, "init");
    if (plan.sampled) {
        EstimateArgs es;
        memset(&es, 0, sizeof es);
        es.rows = index->rows;
        es.dtype = index->dtype;
        es.d = index->d;
        es.inv_norm = index->inv_norm;
        es.exclude = exclude_bits;
        es.inv_tau = inv_tau;
        es.queries = pc.queries;
        es.q_dtype = pc.q_dtype;
        es.qscale = pc.qscale;
        es.b = b;
        es.stride = plan.stride[1];
        es.n_sample = plan.rows[1];
        es.rank = plan.rank[1];
        es.keys = sc.keys;
        es.cap = plan.cap;
        es.theta = sc.theta;
        es.thf = sc.thf;
        es.tickets = sc.flags + 4;
        es.count = estimate_clears ? sc.count : nullptr;
        es.flags = estimate_clears ? sc.flags : nullptr;
        if ((e = launch_estimate(es, s)) != cudaSuccess) return cuda_fail(e, "threshold estimate");
    }
    for (int lv = plan.sampled ? 0 : plan.levels - 1; lv >= 0; --lv) {
        if ((st = run_pass(index, pc, plan, lv, sc, exclude_bits, inv_tau, b, s, sms)) != TT_OK) return st;
        if (lv > 0) {
            e = launch_select_threshold(sc.keys, sc.count, plan.cap, V, plan.rank[lv], sc.theta,
                                        sc.thf, s);
            if (e == cudaSuccess) e = sets_min();
        } else {
            e = launch_select_final(sc.keys, sc.count, plan.cap, V, k, sc.theta, sc.thf, sc.flagged,
                                    sc.flags, out_ids, out_scores, s);
        }
        if (e != cudaSuccess) return cuda_fail(e, "select");
    }
    // Lists the final select could not prove exact are recomputed on the
    // device, in the same stream; with none, every block returns at once.
    ExactArgs ea;
    memset(&ea, 0, sizeof ea);
    ea.rows = index->rows;
    ea.dtype = index->dtype;
    ea.n = index->n;
    ea.d = index->d;
    ea.inv_norm = index->inv_norm;
    ea.exclude = exclude_bits;
    ea.inv_tau = inv_tau;
    ea.queries = pc.queries;
    ea.q_dtype = pc.q_dtype;
    ea.qscale = pc.qscale;
    ea.b = b;
    ea.V = V;
    ea.types = types;
    ea.set_of = types ? sc.set_of : nullptr;
    ea.keys = sc.keys;
    ea.cap = plan.cap;
    ea.k = k;
    ea.theta = sc.theta;
    ea.done = sc.count;
    ea.flagged = sc.flagged;
    ea.flags = sc.flags;
    ea.out_ids = out_ids;
    ea.out_scores = out_scores;
    ea.status = index->dstat;
    ea.seq = seq;
    ea.chunks = exact_chunks(index->n, k, plan.cap);
    e = launch_exact(ea, s, sms);
    if (e != cudaSuccess) return cuda_fail(e, "exact fallback");
    index->tickets_zero_at = sc.flags;
    stats.rescans = -1;  // known once the work has run (tt_last_stats)
    stats.launches = (int)(g_launches.load() - launches0);
    index->last = stats;
    index->last_pending = seq;
    return TT_OK;
}

tt_status tt_score_topk_ex(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                           const uint32_t* exclude_bits, float tau, int32_t k, int32_t* out_ids,
                           float* out_scores, void* stream, const tt_options* options) {
    return score_core(index, queries, q_dtype, b, exclude_bits, tau, k, out_ids, out_scores, stream, options,
                      nullptr, 0, nullptr);
}

tt_status tt_merge_topk(const int32_t* ids, const float* scores, int32_t parts, int32_t b, int32_t k_in,
                        const int64_t* id_offsets, int32_t k_out, int32_t* out_ids, float* out_scores,
                        void* stream) {
    if (b < 0 || parts < 1 || k_in < 1 || k_out < 1) return TT_ERR_INVALID_ARG;
    if (parts > TT_MAX_PARTS || k_in > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    if (k_out > k_in) return TT_ERR_INVALID_ARG;
    if (id_offsets == nullptr) return TT_ERR_INVALID_ARG;
    for (int p = 0; p < parts; ++p)
        if (id_offsets[p] < 0 || id_offsets[p] >= ((int64_t)1 << 31)) return TT_ERR_INVALID_ARG;
    if (b > 0 && (ids == nullptr || scores == nullptr || out_ids == nullptr || out_scores == nullptr))
        return TT_ERR_INVALID_ARG;
    if (!aligned(ids, 4) || !aligned(scores, 4) || !aligned(out_ids, 4) || !aligned(out_scores, 4))
        return TT_ERR_INVALID_ARG;
    if (b == 0) return TT_OK;
    tt_status st;
    if ((st = check_device_ptr(ids, "ids")) != TT_OK) return st;
    if ((st = check_device_ptr(scores, "scores")) != TT_OK) return st;
    if ((st = check_device_ptr(out_ids, "out_ids")) != TT_OK) return st;
    if ((st = check_device_ptr(out_scores, "out_scores")) != TT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t m = (int64_t)parts * k_in;
    uint64_t* scratch = nullptr;
    if (m > merge_smem_keys()) {
        // keys of the lists that do not fit in shared memory, stream-ordered
        TT_CUDA(cudaMallocAsync(reinterpret_cast<void**>(&scratch), (size_t)b * m * sizeof(uint64_t), s),
                "merge scratch");
    }
    cudaError_t e = launch_merge(ids, scores, parts, b, k_in, id_offsets, k_out, scratch, out_ids,
                                 out_scores, s);
    if (scratch) cudaFreeAsync(scratch, s);
    if (e != cudaSuccess) return cuda_fail(e, "merge");
    return TT_OK;
}

// ---------------------------------------------------------------------------
// in-batch sampled softmax
// ---------------------------------------------------------------------------
static tt_status softmax_sizes(int32_t b, int32_t nc, int32_t d, bool with_ids) {
    if (b < 0 || nc < b) return TT_ERR_INVALID_ARG;
    if (d <= 0) return TT_ERR_INVALID_ARG;
    if (d % 16 != 0 || d > TT_MAX_D || !softmax_supported(d)) return TT_ERR_UNSUPPORTED;
    if (with_ids && nc > (1 << 28)) return TT_ERR_UNSUPPORTED;
    return TT_OK;
}

tt_status tt_inbatch_softmax_workspace(int32_t b, int32_t nc, int32_t d, int32_t with_item_ids, size_t* bytes) {
    if (bytes == nullptr) return TT_ERR_INVALID_ARG;
    tt_status st = softmax_sizes(b, nc, d, with_item_ids != 0);
    if (st != TT_OK) return st;
    *bytes = softmax_plan(b, nc, d, with_item_ids != 0, sm_count_current()).bytes;
    return TT_OK;
}

tt_status tt_inbatch_softmax(const void* users, const void* items, tt_dtype dtype, int32_t b, int32_t nc,
                             int32_t d, float tau, const float* logq, const int64_t* item_ids,
                             const uint8_t* valid, float* lse, float* loss, float* mean, void* workspace,
                             size_t workspace_bytes, void* stream) {
    // ---------------- host-side validation (no device calls) ----------------
    if (dtype != TT_BF16) return valid_index_dtype(dtype) ? TT_ERR_UNSUPPORTED : TT_ERR_INVALID_ARG;
    tt_status st = softmax_sizes(b, nc, d, item_ids != nullptr);
    if (st != TT_OK) return st;
    if (!(tau > 0.0f) || !isfinite(tau)) return TT_ERR_INVALID_ARG;
    if (mean == nullptr || workspace == nullptr) return TT_ERR_INVALID_ARG;
    if (b > 0 && (users == nullptr || items == nullptr || lse == nullptr || loss == nullptr))
        return TT_ERR_INVALID_ARG;
    if (!aligned(users, 16) || !aligned(items, 16) || !aligned(logq, 4) || !aligned(item_ids, 8) ||
        !aligned(lse, 4) || !aligned(loss, 4) || !aligned(mean, 4) || !aligned(workspace, 256))
        return TT_ERR_INVALID_ARG;
    const int sms = sm_count_current();
    const SoftmaxPlan pl = softmax_plan(b, nc, d, item_ids != nullptr, sms);
    if (workspace_bytes < pl.bytes) {
        snprintf(g_last_error, sizeof g_last_error, "workspace of %zu bytes, need %zu", workspace_bytes, pl.bytes);
        return TT_ERR_INVALID_ARG;
    }
    // ---------------- device checks ----------------
    if ((st = check_device_ptr(users, "users")) != TT_OK) return st;
    if ((st = check_device_ptr(items, "items")) != TT_OK) return st;
    if ((st = check_device_ptr(logq, "logq")) != TT_OK) return st;
    if ((st = check_device_ptr(item_ids, "item_ids")) != TT_OK) return st;
    if ((st = check_device_ptr(valid, "valid")) != TT_OK) return st;
    if ((st = check_device_ptr(lse, "lse")) != TT_OK) return st;
    if ((st = check_device_ptr(loss, "loss")) != TT_OK) return st;
    if ((st = check_device_ptr(mean, "mean")) != TT_OK) return st;
    if ((st = check_device_ptr(workspace, "workspace")) != TT_OK) return st;
    CUtensorMap tm_users, tm_items;
    memset(&tm_users, 0, sizeof tm_users);
    memset(&tm_items, 0, sizeof tm_items);
    if (b > 0) {
        // with item ids the tensor cores read the bin-order copies in the workspace
        const void* u_src = item_ids ? static_cast<const uint8_t*>(workspace) + pl.off_users_s : users;
        const void* v_src = item_ids ? static_cast<const uint8_t*>(workspace) + pl.off_items_s : items;
        if (!bf16_tile_tensor_map(u_src, b, d, d, 128, &tm_users)) return TT_ERR_CUDA;
        if (!bf16_tile_tensor_map(v_src, nc, d, d, pl.tile_cols, &tm_items)) return TT_ERR_CUDA;
    }
    cudaError_t e = launch_softmax(pl, tm_users, tm_items, users, items, b, nc, d, tau, logq, item_ids, valid, lse,
                                   loss, mean, workspace, static_cast<cudaStream_t>(stream), sms);
    if (e != cudaSuccess) return cuda_fail(e, "in-batch softmax");
    return TT_OK;
}

tt_status tt_inbatch_softmax_check(const void* workspace, void* stream) {
    if (workspace == nullptr || !aligned(workspace, 256)) return TT_ERR_INVALID_ARG;
    tt_status st;
    if ((st = check_device_ptr(workspace, "workspace")) != TT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int err = 0;
    TT_CUDA(cudaMemcpyAsync(&err, workspace, sizeof err, cudaMemcpyDeviceToHost, s), "error word readback");
    TT_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    if (err != 0) {
        snprintf(g_last_error, sizeof g_last_error, "device-side wait expired or check failed (code %d)", err);
        return TT_ERR_TIMEOUT;
    }
    return TT_OK;
}

// One result set: rows [start, start + count) of the index, a mask already
// sliced to those rows (or null), ids reported as corpus ids.
static tt_status score_rows(tt_index* index, int64_t start, int64_t count, const void* queries, tt_dtype q_dtype,
                            int32_t b, const uint32_t* mask, float tau, int32_t k, int32_t* out_ids,
                            float* out_scores, cudaStream_t s) {
    const int esize = index->dtype == TT_F32 ? 4 : index->dtype == TT_BF16 ? 2 : 1;
    // a view of the rows that borrows the handle's work memory and status block
    tt_index sub = *index;
    sub.rows = static_cast<const uint8_t*>(index->rows) + start * index->d * esize;
    sub.n = count;
    sub.inv_norm = index->inv_norm ? index->inv_norm + start : nullptr;
    tt_status st = tt_score_topk_ex(&sub, queries, q_dtype, b, mask, tau, k, out_ids, out_scores, s, nullptr);
    tt_index keep = *index;  // the handle keeps its own view of the corpus
    *index = sub;
    index->rows = keep.rows;
    index->n = keep.n;
    index->inv_norm = keep.inv_norm;
    if (st != TT_OK) return st;
    cudaError_t e = launch_offset_ids(out_ids, (int64_t)b * k, start, s);
    if (e != cudaSuccess) return cuda_fail(e, "id offset");
    return TT_OK;
}

// Common host checks of the multi-set calls (no device calls).
static tt_status check_sets(const tt_index* index, int32_t b, int32_t k, int32_t n_sets, const void* queries,
                            const int32_t* out_ids, const float* out_scores) {
    if (!index || b < 0 || k <= 0) return TT_ERR_INVALID_ARG;
    if (k > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    if (n_sets < 1) return TT_ERR_INVALID_ARG;
    if (n_sets > TT_MAX_PARTS) return TT_ERR_UNSUPPORTED;
    if (b > 0 && (queries == nullptr || out_ids == nullptr || out_scores == nullptr)) return TT_ERR_INVALID_ARG;
    if (!aligned(out_ids, 4) || !aligned(out_scores, 4)) return TT_ERR_INVALID_ARG;
    return TT_OK;
}

tt_status tt_score_topk_ranges(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                               const uint32_t* exclude_bits, float tau, int32_t k, int32_t n_ranges,
                               const int64_t* ranges, int32_t* out_ids, float* out_scores, void* stream) {
    tt_status st = check_sets(index, b, k, n_ranges, queries, out_ids, out_scores);
    if (st != TT_OK) return st;
    if (!ranges) return TT_ERR_INVALID_ARG;
    for (int r = 0; r < n_ranges; ++r)
        if (ranges[2 * r] < 0 || ranges[2 * r] > ranges[2 * r + 1] || ranges[2 * r + 1] > index->n)
            return TT_ERR_INVALID_ARG;
    if (!aligned(exclude_bits, 4)) return TT_ERR_INVALID_ARG;
    if (b == 0) return TT_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t per_set = (int64_t)b * k;
    for (int r = 0; r < n_ranges; ++r) {
        const int64_t start = ranges[2 * r], count = ranges[2 * r + 1] - start;
        uint32_t* mask = nullptr;
        if (exclude_bits && count > 0) {
            if ((st = check_device_ptr(exclude_bits, "exclude_bits")) != TT_OK) return st;
            TT_CUDA(cudaMallocAsync(reinterpret_cast<void**>(&mask), (size_t)((count + 31) / 32) * 4, s),
                    "range mask");
            cudaError_t e = launch_mask_slice(exclude_bits, start, count, nullptr, 0, mask, s);
            if (e != cudaSuccess) {
                cudaFreeAsync(mask, s);
                return cuda_fail(e, "range mask");
            }
        }
        st = score_rows(index, start, count, queries, q_dtype, b, mask, tau, k, out_ids + r * per_set,
                        out_scores + r * per_set, s);
        if (mask) cudaFreeAsync(mask, s);
        if (st != TT_OK) return st;
    }
    return TT_OK;
}

tt_status tt_score_topk_types(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                              const uint32_t* exclude_bits, float tau, int32_t k, const uint8_t* types,
                              int32_t n_sets, const int32_t* set_types, int32_t* out_ids, float* out_scores,
                              void* stream) {
    tt_status st = check_sets(index, b, k, n_sets, queries, out_ids, out_scores);
    if (st != TT_OK) return st;
    if (!set_types || (index->n > 0 && !types)) return TT_ERR_INVALID_ARG;
    for (int t = 0; t < n_sets; ++t)
        if (set_types[t] < 0 || set_types[t] > 255) return TT_ERR_INVALID_ARG;
    if (!aligned(exclude_bits, 4)) return TT_ERR_INVALID_ARG;
    // one list per (set, query): their number must stay a modest int
    if ((int64_t)n_sets * b > TT_MAX_SET_LISTS) return TT_ERR_UNSUPPORTED;
    if (b == 0) return TT_OK;
    if (index->n > 0 && (st = check_device_ptr(types, "types")) != TT_OK) return st;
    // type -> set; a type asked for twice is scored once and its lists copied
    int8_t set_of[256];
    memset(set_of, -1, sizeof set_of);
    int distinct = 0;
    int first_of[TT_MAX_PARTS];
    for (int t = 0; t < n_sets; ++t) {
        if (set_of[set_types[t]] < 0) set_of[set_types[t]] = (int8_t)distinct++;
        first_of[t] = set_of[set_types[t]];
    }
    // the distinct sets' lists go to the front of the output, in first-seen order
    st = score_core(index, queries, q_dtype, b, exclude_bits, tau, k, out_ids, out_scores, stream, nullptr,
                    types, distinct, set_of);
    if (st != TT_OK) return st;
    // move each requested set to its place (from the back, so that no list is
    // overwritten before it is read: set t's source is at index first_of[t] <= t)
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t per_set = (size_t)b * k;
    for (int t = n_sets - 1; t >= 0; --t) {
        if (first_of[t] == t) continue;
        TT_CUDA(cudaMemcpyAsync(out_ids + t * per_set, out_ids + first_of[t] * per_set, per_set * 4,
                                cudaMemcpyDeviceToDevice, s), "set copy");
        TT_CUDA(cudaMemcpyAsync(out_scores + t * per_set, out_scores + first_of[t] * per_set, per_set * 4,
                                cudaMemcpyDeviceToDevice, s), "set copy");
    }
    return TT_OK;
}

tt_status tt_score_topk(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                        const uint32_t* exclude_bits, float tau, int32_t k, int32_t* out_ids,
                        float* out_scores, void* stream) {
    return tt_score_topk_ex(index, queries, q_dtype, b, exclude_bits, tau, k, out_ids, out_scores,
                            stream, nullptr);
}

// Host memory of the process (pageable or pinned), never device memory.
static bool host_memory(const void* p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return true;  // not known to CUDA: ordinary pageable memory
    }
    return attr.type == cudaMemoryTypeUnregistered || attr.type == cudaMemoryTypeHost;
}

tt_status tt_score_topk_host(tt_index* index, const void* host_queries, tt_dtype q_dtype, int32_t b,
                             int32_t normalize, tt_dtype norm_dtype, const uint32_t* exclude_bits, float tau,
                             int32_t k, int32_t* host_ids, float* host_scores, void* stream) {
    // ---------------- host-side validation ----------------
    if (!index || b < 0 || k <= 0) return TT_ERR_INVALID_ARG;
    if (k > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    if (!valid_dtype(q_dtype)) return TT_ERR_INVALID_ARG;
    if (normalize && !valid_dtype(norm_dtype)) return TT_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau)) return TT_ERR_INVALID_ARG;
    if (b > 0 && (host_queries == nullptr || host_ids == nullptr || host_scores == nullptr))
        return TT_ERR_INVALID_ARG;
    if (b == 0) return TT_OK;
    if (!host_memory(host_queries) || !host_memory(host_ids) || !host_memory(host_scores)) {
        snprintf(g_last_error, sizeof g_last_error, "tt_score_topk_host takes host buffers");
        return TT_ERR_INVALID_ARG;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != index->device) {
        snprintf(g_last_error, sizeof g_last_error, "index was made on device %d, current is %d",
                 index->device, dev);
        return TT_ERR_INVALID_ARG;
    }
    tt_status st = report_pending(index);
    if (st != TT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int d = index->d;
    const size_t q_bytes = (size_t)b * d * (q_dtype == TT_F32 ? 4 : 2);
    const size_t n_bytes = normalize ? (size_t)b * d * (norm_dtype == TT_F32 ? 4 : 2) : 0;
    const size_t o_bytes = (size_t)b * k * 4;
    const size_t o_q = 0, o_n = align_up(q_bytes, 256), o_ids = align_up(o_n + n_bytes, 256),
                 o_sc = align_up(o_ids + o_bytes, 256), total = align_up(o_sc + o_bytes, 256);
    if ((st = grow_block(index, &index->io, &index->io_bytes, total, s, "host staging allocation")) != TT_OK)
        return st;
    uint8_t* io = static_cast<uint8_t*>(index->io);
    TT_CUDA(cudaMemcpyAsync(io + o_q, host_queries, q_bytes, cudaMemcpyHostToDevice, s), "queries to device");
    const void* q_dev = io + o_q;
    tt_dtype q_dt = q_dtype;
    if (normalize) {
        // the model normalises the user vector before retrieval (RecsysTwoTowerModel.__call__)
        cudaError_t e = launch_normalize(io + o_q, q_dtype, b, d, io + o_n, norm_dtype, TT_NORM_STORE, s);
        if (e != cudaSuccess) return cuda_fail(e, "query normalize");
        q_dev = io + o_n;
        q_dt = norm_dtype;
    }
    int32_t* d_ids = reinterpret_cast<int32_t*>(io + o_ids);
    float* d_scores = reinterpret_cast<float*>(io + o_sc);
    st = score_core(index, q_dev, q_dt, b, exclude_bits, tau, k, d_ids, d_scores, stream, nullptr, nullptr, 0,
                    nullptr);
    if (st != TT_OK) return st;
    TT_CUDA(cudaMemcpyAsync(host_ids, d_ids, o_bytes, cudaMemcpyDeviceToHost, s), "ids to host");
    TT_CUDA(cudaMemcpyAsync(host_scores, d_scores, o_bytes, cudaMemcpyDeviceToHost, s), "scores to host");
    TT_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    return report_pending(index);  // this search's own expired wait, if any
}

}  // extern "C"
