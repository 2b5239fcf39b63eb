// tt_noalloc.cu - tt_score_topk_noalloc: the exact top-k search for callers
// that cannot allocate device memory.
//
// Some programs are not allowed to call cudaMalloc once they are running:
// a serving process whose memory pool reserved the GPU at start-up (an extra
// cudaMalloc there fails or fragments the pool), or a latency-bound loop in
// which cudaMalloc/cudaFree would stall every stream on the device. The
// regular entry point keeps its work buffers in the index handle and grows
// them with cudaMalloc. This variant allocates nothing: its work buffers live
// in one fixed array in device memory that the library declares at file
// scope, so the memory is set aside when the library's code is loaded onto a
// GPU and stays reserved there until the process exits.
//
// Limits and rules:
//   - the array holds TT_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU; a call whose
//     work buffers would not fit (about 128 KiB per query, so up to 255
//     queries per call) is rejected with TT_ERR_UNSUPPORTED;
//   - all calls on a GPU share the one array: calls that overlap on the GPU
//     (from two streams or two host threads at once) race and corrupt each
//     other's results; the caller must order them;
//   - the array keeps whatever the last call left in it; every call first
//     resets the counters and thresholds it relies on;
//   - the first call on each GPU looks up the array's device address (with
//     that GPU current); make that first call before any stream capture;
//   - like tt_score_topk the call only enqueues its work on the stream and
//     returns; it has no handle to report a device-side timeout through, so
//     a search whose bounded wait expired leaves id -1 and score NaN in every
//     output entry.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "../../include/tt.h"
#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int kMaxDevices = 64;

// The work buffers of tt_score_topk_noalloc. In host code this name is only a
// stand-in for the symbol; kernels get the device address found by
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Status text for tt_last_error().
void noalloc_error(const char* fmt_msg) { set_last_error_message(fmt_msg); }

// Device (or managed) memory of the current device; no allocation involved.
bool on_device(const void* p, int dev) {
    if (p == nullptr) return true;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) &&
           attr.device == dev;
}

// Device address of the array on the current device (looked up once per device).
tt_status noalloc_base(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return TT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            char msg[160];
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the no-alloc work array: %s",
                     cudaGetErrorString(e));
            noalloc_error(msg);
            return TT_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return TT_OK;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace tt

using namespace tt;

extern "C" {

tt_status tt_score_topk_noalloc(const void* rows, tt_dtype dtype, int64_t n, int32_t d,
                                const float* inv_norm, const void* queries, tt_dtype q_dtype,
                                int32_t b, const uint32_t* exclude_bits, float tau, int32_t k,
                                int32_t* out_ids, float* out_scores, void* stream) {
    // ---- host-side checks, before any device call ----
    if (n < 0 || b < 0 || k <= 0) return TT_ERR_INVALID_ARG;
    if (n > TT_MAX_N || k > TT_MAX_K) return TT_ERR_UNSUPPORTED;
    if (d <= 0) return TT_ERR_INVALID_ARG;
    if (d % 16 != 0 || d > TT_MAX_D) return TT_ERR_UNSUPPORTED;
    if (dtype != TT_F32 && dtype != TT_BF16) return TT_ERR_INVALID_ARG;
    if (q_dtype != TT_F32 && q_dtype != TT_BF16) return TT_ERR_INVALID_ARG;
    if (!(tau > 0.0f) || !isfinite(tau)) return TT_ERR_INVALID_ARG;
    if (b > 0 && (queries == nullptr || out_ids == nullptr || out_scores == nullptr))
        return TT_ERR_INVALID_ARG;
    if (n > 0 && rows == nullptr) return TT_ERR_INVALID_ARG;
    if ((uintptr_t)rows % 16 || (uintptr_t)queries % 16 || (uintptr_t)out_ids % 4 ||
        (uintptr_t)out_scores % 4 || (uintptr_t)exclude_bits % 4 || (uintptr_t)inv_norm % 4)
        return TT_ERR_INVALID_ARG;
    if (dtype == TT_F32 && d > 256) return TT_ERR_UNSUPPORTED;
    const bool tc_possible = dtype == TT_BF16 && d >= 64 && tensor_pass_max_nq(d, 2) > 0;
    const int path = (tc_possible && b > 8) ? 2 : 1;
    Plan plan;
    tt_status st = make_plan(n, k, nullptr, path == 1 && b <= 8, &plan);
    if (st != TT_OK) return st;
    const int cap = plan.cap;
    int nq = 0, q_tiles = 1;
    if (path == 2) {
        const int max_nq = tensor_pass_max_nq(d, 2);
        q_tiles = (b + max_nq - 1) / max_nq;
        nq = ((b + q_tiles - 1) / q_tiles + 31) / 32 * 32;  // whole 32-column chunks
        if (nq > max_nq) nq = max_nq;
    }
    const int b_pad = (path == 2 ? q_tiles * nq : b) + 64;
    const bool need_qcast = path == 2 && q_dtype == TT_F32;
    // layout inside the static array
    const size_t o_keys = 0;
    const size_t o_count = up256(o_keys + (size_t)b * cap * 8);
    const size_t o_theta = up256(o_count + (size_t)b_pad * 4);
    const size_t o_thf = up256(o_theta + (size_t)b_pad * 8);
    const size_t o_flagged = up256(o_thf + (size_t)b_pad * 4);
    const size_t o_flags = up256(o_flagged + (size_t)b_pad * 4);
    const size_t o_q = up256(o_flags + 64);
    const size_t total = up256(o_q + (need_qcast ? (size_t)b * d * 2 : 0));
    if (total > (size_t)TT_NOALLOC_SCRATCH_BYTES) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "tt_score_topk_noalloc: b=%d needs %zu bytes of work memory, the fixed array "
                 "holds %d bytes (about %d queries per call at most)",
                 b, total, TT_NOALLOC_SCRATCH_BYTES, TT_NOALLOC_SCRATCH_BYTES / (cap * 8 + 64));
        noalloc_error(msg);
        return TT_ERR_UNSUPPORTED;
    }
    if (b == 0) return TT_OK;

    // ---- device ----
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        noalloc_error("tt_score_topk_noalloc: no current CUDA device");
        return TT_ERR_CUDA;
    }
    if (!on_device(rows, dev) || !on_device(inv_norm, dev) || !on_device(queries, dev) ||
        !on_device(exclude_bits, dev) || !on_device(out_ids, dev) || !on_device(out_scores, dev)) {
        noalloc_error("tt_score_topk_noalloc: every pointer must be device memory of the current GPU");
        return TT_ERR_INVALID_ARG;
    }
    void* base_v = nullptr;
    if ((st = noalloc_base(dev, &base_v)) != TT_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(base_v);
    uint64_t* keys = reinterpret_cast<uint64_t*>(base + o_keys);
    uint32_t* count = reinterpret_cast<uint32_t*>(base + o_count);
    uint64_t* theta = reinterpret_cast<uint64_t*>(base + o_theta);
    float* thf = reinterpret_cast<float*>(base + o_thf);
    int32_t* flagged = reinterpret_cast<int32_t*>(base + o_flagged);
    int* flags = reinterpret_cast<int*>(base + o_flags);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    auto launch_failed = [](const char* what, cudaError_t err) {
        char msg[200];
        snprintf(msg, sizeof msg, "tt_score_topk_noalloc %s: %s", what, cudaGetErrorString(err));
        noalloc_error(msg);
        return TT_ERR_CUDA;
    };

    if (n == 0) {
        e = launch_pad(out_ids, out_scores, (int64_t)b * k, s);
        return e == cudaSuccess ? TT_OK : launch_failed("padding", e);
    }
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const float inv_tau = 1.0f / tau;

    const void* q_use = queries;
    int q_dt_use = q_dtype;
    CUtensorMap tm_q;
    if (path == 2) {
        if (need_qcast) {
            __nv_bfloat16* qc = reinterpret_cast<__nv_bfloat16*>(base + o_q);
            e = launch_cast_bf16(static_cast<const float*>(queries), (int64_t)b * d, qc, s);
            if (e != cudaSuccess) return launch_failed("query cast", e);
            q_use = qc;
            q_dt_use = TT_BF16;
        }
        if (!bf16_tile_tensor_map(q_use, b, d, d, nq, &tm_q)) {
            noalloc_error("tt_score_topk_noalloc: query tensor map could not be encoded");
            return TT_ERR_CUDA;
        }
    }
    auto pass = [&](int lv) -> cudaError_t {
        PassArgs a;
        memset(&a, 0, sizeof a);
        a.rows = rows;
        a.dtype = dtype;
        a.n_rows = plan.rows[lv];
        a.stride = plan.stride[lv];
        a.d = d;
        a.inv_norm = inv_norm;
        a.exclude = exclude_bits;
        a.inv_tau = inv_tau;
        a.queries = q_use;
        a.q_dtype = q_dt_use;
        a.b = b;
        a.theta = theta;
        a.thf = thf;
        a.count = count;
        a.keys = keys;
        a.cap = cap;
        a.err = flags + 1;
        a.defer = (plan.sampled && lv == 0) ? 1 : 0;  // the pass right after the one-sample estimate
        if (path == 2) {
            CUtensorMap tm_rows;
            if (!bf16_tile_tensor_map(rows, a.n_rows, d, a.stride * d, 128, &tm_rows))
                return cudaErrorInvalidValue;
            return launch_tensor_pass(a, tm_rows, tm_q, nq, s, sms);
        }
        return launch_stream_pass(a, s, sms);
    };

    // The array holds the previous call's leftovers: counters, thresholds and
    // flags are reset first, in the stream, before anything reads them.
    e = launch_init(count, theta, thf, KEY_MIN, b, b_pad, flags, s);
    if (e != cudaSuccess) return launch_failed("init", e);
    if (plan.sampled) {
        EstimateArgs es;
        memset(&es, 0, sizeof es);
        es.rows = rows;
        es.dtype = dtype;
        es.d = d;
        es.inv_norm = inv_norm;
        es.exclude = exclude_bits;
        es.inv_tau = inv_tau;
        es.queries = q_use;
        es.q_dtype = q_dt_use;
        es.b = b;
        es.stride = plan.stride[1];
        es.n_sample = plan.rows[1];
        es.rank = plan.rank[1];
        es.keys = keys;
        es.cap = cap;
        es.theta = theta;
        es.thf = thf;
        es.tickets = flags + 4;
        e = launch_estimate(es, s);
        if (e != cudaSuccess) return launch_failed("threshold estimate", e);
    }
    for (int lv = plan.sampled ? 0 : plan.levels - 1; lv >= 0; --lv) {
        e = pass(lv);
        if (e != cudaSuccess) return launch_failed("scoring pass", e);
        e = lv > 0 ? launch_select_threshold(keys, count, cap, b, plan.rank[lv], theta, thf, s)
                   : launch_select_final(keys, count, cap, b, k, theta, thf, flagged, flags, out_ids,
                                         out_scores, s);
        if (e != cudaSuccess) return launch_failed("select", e);
    }
    // lists the final select could not prove exact are recomputed on the device
    ExactArgs ea;
    memset(&ea, 0, sizeof ea);
    ea.rows = rows;
    ea.dtype = dtype;
    ea.n = n;
    ea.d = d;
    ea.inv_norm = inv_norm;
    ea.exclude = exclude_bits;
    ea.inv_tau = inv_tau;
    ea.queries = q_use;
    ea.q_dtype = q_dt_use;
    ea.b = b;
    ea.V = b;
    ea.keys = keys;
    ea.cap = cap;
    ea.k = k;
    ea.theta = theta;
    ea.done = count;
    ea.flagged = flagged;
    ea.flags = flags;
    ea.out_ids = out_ids;
    ea.out_scores = out_scores;
    ea.status = nullptr;  // no handle: an expired device wait shows as NaN scores
    ea.chunks = exact_chunks(n, k, cap);
    e = launch_exact(ea, s, sms);
    if (e != cudaSuccess) return launch_failed("exact fallback", e);
    return TT_OK;
}

}  // extern "C"
