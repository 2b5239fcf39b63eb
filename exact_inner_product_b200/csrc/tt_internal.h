// tt_internal.h - host-side interfaces between the C-ABI layer (tt_api.cu)
// and the kernel launchers (k_*.cu). Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tt.h"

namespace tt {

// One scoring pass over one level of the corpus: level row j is corpus row
// j * stride, for j < n_rows. Survivors (key > theta[q]) are appended to
// keys[q * cap + slot], slot = atomicAdd(count[q], 1); slots >= cap are
// counted but not stored.
struct PassArgs {
    const void* rows;          // corpus [n, d] (level rows are a strided view)
    int dtype;                 // TT_F32 / TT_BF16 (corpus)
    int64_t n_rows;            // rows in this level
    int64_t stride;            // corpus rows between consecutive level rows
    int d;
    const float* inv_norm;     // [n] or null (int8 rows: the per-row scales)
    const uint32_t* exclude;   // [ceil(n/32)] or null
    float inv_tau;
    const void* queries;       // [b, d] (int8 rows: the query codes)
    int q_dtype;
    int b;
    const uint64_t* theta;     // [b_pad] threshold keys (KEY_MAX past b)
    const float* thf;          // [b_pad] key_floor(theta), +inf past b
    uint32_t* count;           // [b]
    uint64_t* keys;            // [b * cap]
    int cap;
    int* err;                  // device error word
    const float* qscale;       // [b] query scales of int8 rows, else null
    int withhold_copy;         // test hook (tensor-core pass): skip the first corpus copy
    // Several result sets by candidate type, from one pass (null types: one
    // set). Row j belongs to set s = set_of[types[j]] (-1: to none); its
    // keys go to the virtual query v = s * b + q and must beat theta_v[v];
    // count and keys are indexed by v. theta and thf then hold, per query,
    // the minimum over the sets, for the kernels' first (fast) tests.
    const uint8_t* types;      // [n] or null
    const int8_t* set_of;      // [256]
    const uint64_t* theta_v;   // [n_sets * b]
    int defer;                 // streaming pass right after the one-sample estimate (its thresholds)
};

// Launch `kernel` with programmatic stream serialization: it may start while
// the stream's previous kernel still runs (the kernel then orders its memory
// accesses with pdl_wait(), see tt_device.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The scan plan of a search (tt_api.cu). Level i scans every stride[i]-th
// row; rank[i] (i >= 1): the r-th best key of level i, minus one, is the
// filter threshold of level i - 1. A sampled plan (small batches on the
// streaming scorer: small_batch) has two levels, and its level 1 is scored
// and reduced to the threshold by one launch (launch_estimate).
constexpr int MAX_LEVELS = 4;
struct Plan {
    int levels;
    int64_t stride[MAX_LEVELS];
    int64_t rows[MAX_LEVELS];
    int rank[MAX_LEVELS];
    int cap;
    bool sampled;
};
tt_status make_plan(int64_t n, int32_t k, const tt_options* opt, bool small_batch, Plan* p);

// Set the text tt_last_error() returns on the calling thread.
void set_last_error_message(const char* msg);

// Kernel launch bookkeeping (counts and optional event timing).
void note_launch_begin(int kind, cudaStream_t s);
void note_launch_end(int kind, cudaStream_t s);

// Launchers. Each returns cudaSuccess or the launch error.
cudaError_t launch_normalize(const void* in, int in_dtype, int64_t n, int d, void* out,
                             int out_dtype, int mode, cudaStream_t s);
cudaError_t launch_cast_bf16(const float* in, int64_t count, __nv_bfloat16* out, cudaStream_t s);
// int8 coding of rows (normalised first when `normalise`): codes [n, d],
// scales [n] (see tt_quantize_candidates).
cudaError_t launch_quantize(const void* in, int in_dtype, int64_t n, int d, int8_t* codes, float* scales,
                            bool normalise, cudaStream_t s);
cudaError_t launch_stream_pass(const PassArgs& a, cudaStream_t s, int sm_count);
cudaError_t launch_tensor_pass(const PassArgs& a, const CUtensorMap& tm_rows,
                               const CUtensorMap& tm_queries, int nq_tile, cudaStream_t s,
                               int sm_count);
// Tensor-core pass on SM pairs (b >= 1, bf16 queries in tiles of 256;
// tm_rows with boxes of tensor_pair_box_rows(d) rows).
cudaError_t launch_tensor_pair_pass(const PassArgs& a, const CUtensorMap& tm_rows, cudaStream_t s,
                                    int sm_count);
int tensor_pair_box_rows(int d);
// count[0..b) = 0; theta/thf[0..b) = theta_value; [b, b_pad) = KEY_MAX / +inf;
// flags[0..16) = 0 (flagged lists, error word, estimate tickets).
cudaError_t launch_init(uint32_t* count, uint64_t* theta, float* thf, uint64_t theta_value, int b,
                        int b_pad, int* flags, cudaStream_t s);
// The threshold of a small batch from one sample of the corpus, in one
// launch (k_estimate.cu): level row j = corpus row j * stride (j < n_sample)
// is scored for every query with the streaming scorer's arithmetic; blocks of
// 256 sample rows keep their best `rank` keys per query (in keys[q * cap...]),
// and the last block of each query sets theta[q] = (rank-th best key) - 1, or
// KEY_MIN when fewer were eligible. tickets: [b] counters, zero on entry.
struct EstimateArgs {
    const void* rows;
    int dtype;
    int d;
    const float* inv_norm;
    const uint32_t* exclude;
    float inv_tau;
    const void* queries;  // as the streaming pass reads them (int8: codes)
    int q_dtype;
    const float* qscale;  // int8: query scales
    int b;
    int64_t stride;
    int64_t n_sample;
    int rank;
    uint64_t* keys;       // work keys [b * cap]; blocks' lists at keys[q * cap + g * rank]
    int cap;
    uint64_t* theta;
    float* thf;
    int* tickets;
    // As the search's first kernel, the estimate clears the work memory a
    // separate init kernel clears otherwise: count[q] and flags[0..4)
    // (null: not cleared here). The tickets clear themselves.
    uint32_t* count;
    int* flags;
};
constexpr int ESTIMATE_BLOCK_ROWS = 256;  // sample rows per block: one per thread
constexpr int ESTIMATE_MAX_RANK = 256;    // the sample rank a plan may ask of the estimate
cudaError_t launch_estimate(const EstimateArgs& a, cudaStream_t s);

// Threshold mode: theta_next[q] = (r-th best kept key) - 1, or KEY_MIN when
// fewer than r keys were kept; counts reset to 0.
cudaError_t launch_select_threshold(const uint64_t* keys, uint32_t* count, int cap, int b, int r,
                                    uint64_t* theta_next, float* thf_next, cudaStream_t s);
// Final mode: writes the sorted top-k (ids, scores) of lists whose pass was
// exact; any other list goes to flagged[atomicAdd(flags[0], 1)], with a valid
// lower bound on its k-th best key left in theta, for the exact fallback.
// Skips everything when flags[1] (a device wait expired) is set.
cudaError_t launch_select_final(const uint64_t* keys, uint32_t* count, int cap, int b, int k,
                                uint64_t* theta, float* thf, int32_t* flagged, int* flags,
                                int32_t* out_ids, float* out_scores, cudaStream_t s);

// Written by the device at the end of every search (host-mapped memory of an
// index handle): the error code of an expired device wait (only written when
// there is one; the host clears it once reported), and the number of lists the
// exact fallback recomputed with the sequence number of the call.
struct HostStatus {
    volatile int32_t err;
    int32_t reserved;
    // low 32 bits of the call's sequence number << 32 | lists recomputed, in
    // one store (the host can never see one half of it without the other)
    volatile uint64_t seq_repaired;
};

// The exact fallback scan (k_exact.cu), launched at the end of every search.
struct ExactArgs {
    const void* rows;          // corpus [n, d] (row stride d)
    int dtype;                 // TT_F32 / TT_BF16 / TT_I8
    int64_t n;
    int d;
    const float* inv_norm;     // [n] or null (int8: the per-row scales)
    const uint32_t* exclude;   // [ceil(n/32)] or null
    float inv_tau;
    const void* queries;       // [b, d] as the main passes read them (int8: codes)
    int q_dtype;
    const float* qscale;       // int8: query scales [b]
    int b;                     // queries
    int V;                     // lists (b, or sets * b)
    const uint8_t* types;      // several result sets by type, else null
    const int8_t* set_of;
    uint64_t* keys;            // [V * cap] work keys
    int cap;
    int k;
    const uint64_t* theta;     // [V] lower bounds left by the final select
    uint32_t* done;            // [V] chunk counters, zero on entry
    const int32_t* flagged;    // lists to recompute (flags[0] of them)
    const int* flags;          // [0] flagged lists, [1] error word
    int32_t* out_ids;          // [V, k]
    float* out_scores;
    HostStatus* status;        // device view of the handle's status block, or null
    int64_t seq;
    int chunks;                // corpus chunks per list (exact_chunks)
};
int exact_chunks(int64_t n, int k, int cap);
cudaError_t launch_exact(const ExactArgs& a, cudaStream_t s, int sm_count);

// Merge per-shard top-k lists (see k4_merge); id_offset_host: host array of
// `parts` global-id offsets; scratch: b * parts * k_in keys when parts * k_in
// exceeds merge_smem_keys(), else unused (may be null).
cudaError_t launch_merge(const int32_t* ids, const float* scores, int parts, int b, int k_in,
                         const int64_t* id_offset_host, int k_out, uint64_t* scratch, int32_t* out_ids,
                         float* out_scores, cudaStream_t s);
int merge_smem_keys();
// Tensor maps (built on the host through the driver entry point).
// Tensor-core pass: bf16 boxes of 64 elements x box_rows rows, 128-byte swizzle.
bool bf16_tile_tensor_map(const void* base, int64_t rows, int d, int64_t row_pitch_elems,
                          int box_rows, CUtensorMap* tm);
// int8 codes: boxes of 128 codes (one 128-byte swizzle row) x box_rows rows.
bool i8_tile_tensor_map(const void* base, int64_t rows, int d, int64_t row_pitch_elems, int box_rows,
                        CUtensorMap* tm);
cudaError_t launch_pad(int32_t* out_ids, float* out_scores, int64_t count, cudaStream_t s);
// Exclusion words for rows [start, start + count) of a mask (null: none),
// optionally also excluding rows whose types[j] != want (types null: none).
cudaError_t launch_mask_slice(const uint32_t* in, int64_t start, int64_t count, const uint8_t* types, int want,
                              uint32_t* out, cudaStream_t s);
// ids[i] += offset where ids[i] >= 0.
// In-batch sampled softmax (k_softmax.cu): work split and workspace layout
// (byte offsets of each region; the error word is at offset 0).
struct SoftmaxPlan {
    int tile_cols;  // candidates per tile (rows of one items box)
    int u_tiles, c_tiles, chunks, stages, log2_slots, merge_blocks;
    int sort_tile, sort_tiles0, sort_tiles1;  // bin order (item ids only)
    size_t off_err, off_ticket, off_col, off_numer, off_part, off_keys, off_block_sum, off_block_rows;
    size_t off_perm, off_sbin, off_hist, off_bstart, off_col_s, off_users_s, off_items_s;
    size_t bytes;
};
SoftmaxPlan softmax_plan(int b, int nc, int d, bool item_ids, int sm_count);
bool softmax_supported(int d);
// users [b, d] and items [nc, d] bf16 (16-byte aligned). The tensor cores
// read them through tm_users (boxes of 64 x 128) and tm_items (boxes of
// 64 x tile_cols), which must map, with item ids, the bin-order copies in the
// workspace at off_users_s / off_items_s, else users and items themselves.
cudaError_t launch_softmax(const SoftmaxPlan& pl, const CUtensorMap& tm_users, const CUtensorMap& tm_items,
                           const void* users, const void* items, int b, int nc, int d, float tau, const float* logq,
                           const int64_t* item_ids, const uint8_t* valid, float* lse, float* loss, float* mean,
                           void* workspace, cudaStream_t s, int sm_count);
// Per query, the minimum over n_sets of the virtual thresholds (v = s * b + q):
// theta_min[q], thf_min[q] for q < b; KEY_MAX / +inf for b <= q < b_pad.
cudaError_t launch_sets_min(const uint64_t* theta_v, const float* thf_v, int n_sets, int b, int b_pad,
                            uint64_t* theta_min, float* thf_min, cudaStream_t s);
cudaError_t launch_offset_ids(int32_t* ids, int64_t count, int64_t offset, cudaStream_t s);

// Shared-memory bytes the tensor-core pass needs for a given d and query tile.
// esize: bytes per element of the rows (2 bf16, 1 int8).
int tensor_pass_smem_bytes(int d, int nq_tile, int esize);
int tensor_pass_max_nq(int d, int esize);
int tensor_pair_smem_bytes(int d, int esize);  // -1 when d does not fit (esize: 2 bf16, 1 int8)

}  // namespace tt
