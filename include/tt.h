/*
 * tt.h - exact top-k maximum-inner-product search on NVIDIA B200 (sm_100a).
 *
 * The retrieval step of a two-tower recommender: L2-normalise the candidate
 * corpus once, then for every user (query) vector return the k candidates
 * with the largest dot product, exactly (brute force, no approximation).
 *
 *   x-algorithm recsys_two_tower_model.py:
 *     `_l2_normalize_candidates`  v / sqrt(max(sum v^2, 1e-12))
 *     `forward` / `compute_top_k`  scores = user . post_embeddings^T
 *     `forward` / `mask_and_top_k` excluded candidates never win; sorted top-k
 *   Two-Tower Retrieval at Industrial Scale, TwoTower.score: u @ v.t() / tau
 *   mhtirogla.ai Two-tower retrieval, Code, Towers::top_k: score every item,
 *     stable sort descending (lower index first on equal scores), take k.
 *
 * Conventions for every entry point:
 *   - Data pointers are DEVICE pointers (cudaMalloc'd or torch CUDA tensors)
 *     owned by the caller, 16-byte aligned, rows contiguous (row-major
 *     [rows, d], row stride d elements). Host pointers are rejected with
 *     TT_ERR_INVALID_ARG (except by tt_score_topk_host, which takes host
 *     buffers for the queries and results).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued on it in order.
 *   - Arguments are validated on the host before any device work; a rejected
 *     call has no side effects.
 *   - Errors are reported as tt_status values only; nothing aborts the process.
 *   - bf16 means IEEE binary32 truncated to its upper 16 bits (bfloat16);
 *     conversions to bf16 round to nearest, ties to even.
 */
#ifndef TT_H
#define TT_H

#include <stdint.h>

#if defined(__GNUC__)
#define TT_API __attribute__((visibility("default")))
#else
#define TT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tt_status {
    TT_OK = 0,
    TT_ERR_INVALID_ARG = 1, /* null, host or misaligned pointer; negative size; bad tau; ... */
    TT_ERR_UNSUPPORTED = 2, /* well-formed but outside the kernels' range (see limits below) */
    TT_ERR_CUDA = 3,        /* a CUDA call failed; tt_last_error() has the message */
    TT_ERR_NO_MEMORY = 4,   /* device or pinned-host allocation failed */
    TT_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired; outputs are not valid */
    TT_ERR_INTERNAL = 6     /* reserved (not returned: the exact fallback has no failure mode) */
} tt_status;

typedef enum tt_dtype {
    TT_F32 = 0,
    TT_BF16 = 1,
    TT_I8 = 2 /* int8 codes with one f32 scale per row (tt_quantize_candidates) */
} tt_dtype;

/* How tt_normalize_candidates prepares the corpus. */
typedef enum tt_norm_mode {
    TT_NORM_STORE = 0, /* write normalised rows v_j / norm_j to `out` ([n,d], out_dtype) */
    TT_NORM_FUSED = 1  /* keep rows raw; write inv_norm_j = 1 / norm_j to `out` ([n] f32);
                          scores are multiplied by inv_norm_j inside the scorer */
} tt_norm_mode;

/* Limits. */
#define TT_MAX_D 512        /* d must be a multiple of 16 and at most 512 (f32 corpus: 256) */
#define TT_MAX_K 2048       /* k at most 2048 */
#define TT_MAX_PARTS 64     /* shards merged by one tt_merge_topk call; result sets of one call */
#define TT_MAX_SET_LISTS (1 << 24) /* tt_score_topk_types: n_sets * b at most this */
#define TT_MAX_N 2147483647 /* candidate ids are int32: n < 2^31 */

/* Opaque handle describing a prepared corpus. Owned by the library; release
 * with tt_free. It refers to, but does not own, the caller's corpus buffers,
 * which must stay alive and unchanged while the handle is used. It also owns
 * the device scratch memory of tt_score_topk (grown on demand). A handle must
 * not be used from two host threads at once. */
typedef struct tt_index tt_index;

/*
 * tt_normalize_candidates - row-wise L2 normalisation of a corpus.
 *
 *   norm_j = sqrt(max(sum_i v_ji^2, 1e-12))      (fp32 arithmetic)
 *   TT_NORM_STORE: out[j,i] = v_ji / norm_j, rounded to out_dtype
 *   TT_NORM_FUSED: out[j]   = 1 / norm_j (f32); `in` is left as is
 *
 * (recsys_two_tower_model.py `_l2_normalize_candidates`; the same formula
 * normalises the user vector in `RecsysTwoTowerModel.__call__`, so this call
 * also serves to normalise a batch of queries.)
 *
 * in        device [n, d] rows, in_dtype (TT_F32 or TT_BF16)
 * n         rows, 0 <= n < 2^31 (n = 0 is allowed: nothing to do)
 * d         row width, multiple of 16, 16 <= d <= 512
 * out       device buffer: [n, d] out_dtype (STORE) or [n] f32 (FUSED). For
 *           STORE it may alias `in` when the dtypes match.
 * out_dtype TT_F32 or TT_BF16 (ignored for FUSED)
 * mode      tt_norm_mode
 * stream    cudaStream_t
 * index_out optional: if not NULL, receives a new handle over the prepared
 *           corpus (STORE: rows = out; FUSED: rows = in, inv_norm = out),
 *           which the caller releases with tt_free. If NULL, only the
 *           normalisation is enqueued (e.g. for queries).
 */
TT_API tt_status tt_normalize_candidates(const void* in, tt_dtype in_dtype, int64_t n, int32_t d,
                                  void* out, tt_dtype out_dtype, int32_t mode, void* stream,
                                  tt_index** index_out);

/*
 * tt_quantize_candidates - L2-normalise each row and code it in int8 with
 * one scale per row, for int8 scoring.
 *
 *   w_ji = fl(v_ji / norm_j)   (norm_j as in tt_normalize_candidates, fp32)
 *   scale_j = max(fl(max_i |w_ji| / 127), 1e-12)
 *   code_ji = clip(round_half_even(fl(w_ji / scale_j)), -127, 127)
 *
 * (recsys_two_tower_model.py `forward`, `compute_top_k_int8`: the user rows
 *  are coded this way and the candidate index arrives as int8 codes with one
 *  scale per candidate; the pages do not show how those are made, and this
 *  call applies the same scheme to the normalised candidate rows.)
 *
 * in          device [n, d] rows, in_dtype (TT_F32 or TT_BF16)
 * n, d        as in tt_normalize_candidates
 * out_codes   device [n, d] int8 (caller-owned)
 * out_scales  device [n] f32 (caller-owned)
 * stream      cudaStream_t
 * index_out   optional: receives a handle over (out_codes, out_scales),
 *             dtype TT_I8, released with tt_free
 *
 * Errors as tt_normalize_candidates; out_codes and out_scales must be
 * 16-byte and 4-byte aligned device pointers.
 */
TT_API tt_status tt_quantize_candidates(const void* in, tt_dtype in_dtype, int64_t n, int32_t d,
                                        int8_t* out_codes, float* out_scales, void* stream,
                                        tt_index** index_out);

/*
 * tt_index_wrap - a handle over a corpus that is already prepared (rows
 * normalised and stored, or raw rows plus their f32 inv_norm, or int8 codes
 * plus their f32 scales), e.g. loaded from a checkpoint. No device work.
 * rows: device [n, d] dtype; inv_norm: device [n] f32 or NULL (for TT_I8
 * rows: the per-row scales, required). Limits as for tt_normalize_candidates.
 */
TT_API tt_status tt_index_wrap(const void* rows, tt_dtype dtype, int64_t n, int32_t d,
                        const float* inv_norm, tt_index** index_out);

/*
 * tt_score_topk - exact top-k by inner product for a batch of queries.
 *
 *   s_bj = fl(dot_bj * c_j),  c_j = fl(inv_norm_j * fl(1/tau))  (inv_norm_j = 1
 *          unless the handle was prepared with TT_NORM_FUSED)
 *   dot_bj = sum_i q_bi * v_ji with fp32 accumulation
 *   int8 handle (TT_I8): each query row is coded as in tt_quantize_candidates
 *   but without normalisation (codes u8_b, scale us_b), and
 *   s_bj = fl(fl(fl(acc_bj) * us_b) * c_j), c_j = fl(scale_j * fl(1/tau)),
 *   acc_bj = sum_i u8_bi * v8_ji exactly in int32
 *   (recsys_two_tower_model.py `compute_top_k_int8`)
 *   For each query: the k eligible candidates with the largest s_bj, sorted by
 *   s descending; equal scores are ordered by ascending id. Candidates whose
 *   exclusion bit is set never appear. When fewer than k candidates are
 *   eligible, the remaining slots hold id -1 and score -INFINITY.
 *
 * (recsys_two_tower_model.py `forward`: compute_top_k, mask_and_top_k,
 *  local_top_k with k_actual = min(k, N); TwoTower.score divides by tau.)
 *
 * The result is exact: the kernels keep fp32 scores and select by a total
 * order on (score, id). The filtered passes are checked on the device; a
 * list they cannot prove exact is recomputed, still on the device and in the
 * same stream, by an exact scan with no capacity limit (launched at the end
 * of every search; it returns at once when nothing needs it).
 *
 * index        handle from tt_normalize_candidates or tt_index_wrap
 * queries      device [b, d], q_dtype. Queries are used as given (normalise
 *              them first if the model expects unit vectors). On the tensor-
 *              core path an f32 query batch is rounded to bf16 first; an f32
 *              corpus or b <= 8 keeps f32 queries exactly.
 * q_dtype      TT_F32 or TT_BF16
 * b            number of queries, b >= 0 (b = 0: nothing to do)
 * exclude_bits device uint32 words, ceil(n/32) of them, or NULL for none.
 *              Bit (j & 31) of word (j >> 5) set = candidate j excluded.
 * tau          temperature, finite and > 0 (1 = plain inner product)
 * k            1 <= k <= 2048
 * out_ids      device [b, k] int32
 * out_scores   device [b, k] f32
 * stream       cudaStream_t
 *
 * Asynchronous: TT_OK means the arguments were valid and the whole search
 * is enqueued on `stream`; the outputs are complete when the stream reaches
 * that point. The host never waits for the device here. Calls on one handle
 * must be issued on one stream (or ordered by the caller), because they
 * share the handle's work memory.
 * Device-side timeouts: if a bounded wait of the search expires (a correct
 * run never does), every entry of its outputs becomes (id -1, score NaN), and
 * the next call on the handle, or tt_index_check, returns TT_ERR_TIMEOUT
 * (once, without enqueueing anything).
 */
TT_API tt_status tt_score_topk(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                        const uint32_t* exclude_bits, float tau, int32_t k, int32_t* out_ids,
                        float* out_scores, void* stream);

/* Path selection and test hooks for tt_score_topk_ex. Zero-initialise, then
 * set fields; tt_score_topk uses all zeros. */
typedef struct tt_options {
    int32_t path;           /* 0 auto; 1 CUDA-core streaming scorer; 2 tensor-core scorer
                               (one SM per tile); 3 tensor-core scorer on SM pairs */
    int32_t rank_scale_pct; /* 0 = 100. Scales the ranks used to set the estimated
                               thresholds (test hook: < 100 provokes rescans) */
    int32_t force_levels;   /* 0 auto; > 0 = number of levels (1 = single pass) */
    int32_t cap;            /* 0 auto (16384); candidate buffer per query, power of 2,
                               256..16384 (test hook: small values provoke overflow) */
    int32_t withhold_copy;  /* test hook, 0 = off. 1: the single-SM tensor-core pass
                               (path 2) never issues its first corpus copy, so the wait
                               for it gives up after its time limit (about 2 s) and the
                               call returns TT_ERR_TIMEOUT; the device and the handle
                               stay usable. Exercises the bounded-wait failure path. */
} tt_options;

TT_API tt_status tt_score_topk_ex(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                           const uint32_t* exclude_bits, float tau, int32_t k, int32_t* out_ids,
                           float* out_scores, void* stream, const tt_options* options);

/* What the last tt_score_topk on a handle did. */
typedef struct tt_stats {
    int32_t path;            /* 1 streaming, 2 tensor core, 3 tensor core on SM pairs */
    int32_t levels;          /* scoring passes in the plan (1 = single pass) */
    int32_t rescans;         /* lists the exact fallback recomputed; -1 while the
                                search's work has not completed yet */
    int32_t launches;        /* kernels launched by the call */
    int64_t level_rows[4];   /* rows scanned per level, finest first */
    int64_t level_stride[4]; /* corpus-row stride per level */
    int32_t cap;             /* candidate buffer per query */
    int32_t sampled;         /* 1: level 1 is a one-launch sample estimate of the
                                threshold (small batches on the streaming scorer),
                                not a filtered pass; 0 otherwise */
} tt_stats;

TT_API tt_status tt_last_stats(const tt_index* index, tt_stats* out);

/*
 * tt_index_check - wait for the work enqueued on `stream` and report whether
 * a device-side wait of a search on this handle expired (TT_ERR_TIMEOUT,
 * reported once; that search's outputs hold id -1 and score NaN) or not
 * (TT_OK). TT_ERR_CUDA if the stream itself failed.
 */
TT_API tt_status tt_index_check(tt_index* index, void* stream);

/*
 * tt_score_topk_host - the search from host buffers to host buffers: copies
 * the b x d queries to the device, optionally L2-normalises them there
 * (normalize != 0, into norm_dtype, as the model normalises the user vector in
 * RecsysTwoTowerModel.__call__), runs tt_score_topk against the index resident
 * in device memory, and copies (ids, scores) back. Synchronous: it returns
 * once host_ids and host_scores hold the result.
 *
 * host_queries  HOST [b, d] q_dtype (pinned memory makes the copy faster;
 *               pageable memory works)
 * normalize     0: score the queries as given; else normalise them first
 * norm_dtype    TT_F32 or TT_BF16: the dtype the normalised queries are kept in
 * exclude_bits  DEVICE mask words as in tt_score_topk, or NULL
 * host_ids      HOST [b, k] int32; host_scores HOST [b, k] f32
 * The device staging buffers belong to the handle (grown on demand).
 * Errors as tt_score_topk; TT_ERR_TIMEOUT when this search's own device
 * wait expired.
 */
TT_API tt_status tt_score_topk_host(tt_index* index, const void* host_queries, tt_dtype q_dtype, int32_t b,
                                    int32_t normalize, tt_dtype norm_dtype, const uint32_t* exclude_bits,
                                    float tau, int32_t k, int32_t* host_ids, float* host_scores, void* stream);

/*
 * tt_plan - the scan plan tt_score_topk would use for a corpus of n rows and
 * a given k (host only, no device work). Level 0 is the whole corpus; level i
 * scans every (61^i)-th row. The deepest level keeps every key; the r-th best
 * key of level i (ranks[i], i >= 1) sets the filter threshold of level i-1.
 * Arrays receive up to 4 entries. Any output pointer may be NULL.
 * Errors as tt_score_topk for n, k and options.
 */
TT_API tt_status tt_plan(int64_t n, int32_t k, const tt_options* options, int32_t* levels, int64_t* rows,
                  int64_t* strides, int32_t* ranks, int32_t* cap);

/*
 * tt_merge_topk - the top-k of a corpus split into row shards, from the
 * shards' own top-k lists (e.g. one shard per GPU: tt_score_topk on each,
 * then an all-gather of the lists, then this call on every GPU or on one).
 *
 * (recsys_two_tower_model.py `forward` shards the corpus over devices on the
 *  `expert` axis and combines the per-device scores before `top_k_by_key`;
 *  here only each shard's top-k crosses devices, and this call combines them.)
 *
 * ids, scores  device [parts, b, k_in] int32 / f32: part p's list for each
 *              query, in tt_score_topk's output form (local ids within the
 *              shard, sorted or not; id -1 = padding, ignored)
 * parts        1 <= parts <= TT_MAX_PARTS
 * b            queries, b >= 0
 * k_in         entries per list, 1 <= k_in <= TT_MAX_K
 * id_offsets   HOST [parts]: global id of the shard's local id 0 (>= 0);
 *              local id + offset must stay below 2^31; shards must be
 *              disjoint (equal global ids are not merged into one)
 * k_out        1 <= k_out <= k_in: entries per query in the result
 * out_ids,     device [b, k_out]: the k_out best (score, global id) of the
 * out_scores   union, sorted by score descending then id ascending; padded
 *              with (-1, -INFINITY). Equal to the single-corpus result when
 *              every shard's list is that shard's exact top-k_in.
 * stream       cudaStream_t; the call is asynchronous (no synchronisation)
 *
 * Errors: TT_ERR_INVALID_ARG (bad sizes, pointers, offsets),
 * TT_ERR_UNSUPPORTED (parts or k beyond the limits), TT_ERR_CUDA.
 */
TT_API tt_status tt_merge_topk(const int32_t* ids, const float* scores, int32_t parts, int32_t b,
                               int32_t k_in, const int64_t* id_offsets, int32_t k_out,
                               int32_t* out_ids, float* out_scores, void* stream);

/*
 * tt_score_topk_ranges - one top-k list per candidate range, from one call.
 *
 * (recsys_two_tower_model.py `forward`, the `dataset_ranges` path: for each
 *  (start, end) the candidate slice [start, end) gets its own top-k, with
 *  indices offset by start.)
 *
 * For range r = [ranges[2r], ranges[2r+1]) the result is exactly
 * tt_score_topk over the rows of that range (same scores, same order and
 * padding), with ids reported as corpus ids. Ranges may be empty or
 * overlap. Each range is scanned once, so disjoint ranges together read
 * each row at most once.
 *
 * ranges    HOST int64 [n_ranges * 2]: 0 <= start <= end <= n
 * n_ranges  1 <= n_ranges <= TT_MAX_PARTS
 * out_ids, out_scores  device [n_ranges, b, k]
 * other arguments, the exactness, the errors and the asynchronous
 * completion as tt_score_topk.
 */
TT_API tt_status tt_score_topk_ranges(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                                      const uint32_t* exclude_bits, float tau, int32_t k, int32_t n_ranges,
                                      const int64_t* ranges, int32_t* out_ids, float* out_scores,
                                      void* stream);

/*
 * tt_score_topk_types - one top-k list per candidate type, from one call.
 *
 * (recsys_two_tower_model.py `forward`, the `target_dataset_types` path: for
 *  each target type, `mask_and_top_k` over the candidates whose dataset type
 *  matches.)
 *
 * Set s keeps only candidates j with types[j] == set_types[s] (and not
 * excluded by exclude_bits); the result is exactly tt_score_topk with that
 * combined mask. All sets come from the same passes over the corpus: every
 * score is computed once, and a candidate that beats its query's loosest
 * set threshold is kept in the list of its own type's set. A type asked for
 * twice is scored once and its lists copied. The work buffers hold n_sets * b
 * lists.
 *
 * types      device uint8 [n]: the type of every candidate
 * set_types  HOST int32 [n_sets], each 0..255
 * n_sets     1 <= n_sets <= TT_MAX_PARTS, and n_sets * b <= TT_MAX_SET_LISTS
 * out_ids, out_scores  device [n_sets, b, k]
 * other arguments, the exactness, the errors and the asynchronous
 * completion as tt_score_topk.
 */
TT_API tt_status tt_score_topk_types(tt_index* index, const void* queries, tt_dtype q_dtype, int32_t b,
                                     const uint32_t* exclude_bits, float tau, int32_t k, const uint8_t* types,
                                     int32_t n_sets, const int32_t* set_types, int32_t* out_ids,
                                     float* out_scores, void* stream);

/*
 * tt_inbatch_softmax - the in-batch sampled-softmax training loss, fused:
 * logits, masks, log-sum-exp and cross-entropy in one tensor-core pass that
 * never writes the b x nc logit matrix.
 *
 * ("Two-Tower Retrieval at Industrial Scale", section 3, In-batch sampled
 *  softmax, `in_batch_loss`; section 4, The LogQ Correction,
 *  `corrected_in_batch_loss`; x-algorithm recsys_two_tower_model.py
 *  `compute_retrieval_loss`, in-batch and global negatives.)
 *
 * Row i (i < b) is a user u_i whose positive is candidate row i; candidates
 * b..nc-1 are negatives shared by every row. For every pair
 *     l_ij = (u_i . v_j) / tau - logq_j
 * (the correction on every column, the positive included). Column j enters
 * row i's denominator when valid[j] and it is not an accidental hit: j == i,
 * or item_ids[j] != item_ids[i]. Then
 *     lse_i  = log sum_j exp(l_ij)          (-inf if no column enters)
 *     loss_i = lse_i - l_ii for valid rows (valid[i]), 0 otherwise
 *     mean   = sum of loss_i over valid rows / their number (0 if none)
 * The dot products are exact products of the bf16 inputs accumulated in
 * fp32 on the tensor cores; the exponentials are single-precision.
 *
 * users     device bf16 [b, d]
 * items     device bf16 [nc, d], b <= nc
 * dtype     TT_BF16 (other types: TT_ERR_UNSUPPORTED; cast first)
 * d         multiple of 16, 64 <= d <= TT_MAX_D (zero-pad narrower rows)
 * tau       > 0, finite
 * logq      device f32 [nc] (finite), or NULL for no correction
 * item_ids  device int64 [nc], or NULL for no accidental-hit mask
 *           (with ids, nc is at most 2^28)
 * valid     device uint8 [nc] (0 = padding), or NULL when every row is valid
 * lse, loss device f32 [b]; mean device f32 [1]
 * workspace device memory of at least tt_inbatch_softmax_workspace bytes,
 *           256-byte aligned, owned by the caller, not shared with another
 *           call in flight (with item ids it also holds copies of users and
 *           items in an order grouped by a hash of the id: about 2·d bytes
 *           per user and per candidate; the results do not depend on it)
 *
 * Asynchronous: the work is enqueued on `stream` and the call returns. If a
 * bounded device-side wait expires (which a correct run never does), every
 * output is NaN and tt_inbatch_softmax_check then returns TT_ERR_TIMEOUT.
 */
TT_API tt_status tt_inbatch_softmax_workspace(int32_t b, int32_t nc, int32_t d, int32_t with_item_ids,
                                              size_t* bytes);
TT_API tt_status tt_inbatch_softmax(const void* users, const void* items, tt_dtype dtype, int32_t b, int32_t nc,
                                    int32_t d, float tau, const float* logq, const int64_t* item_ids,
                                    const uint8_t* valid, float* lse, float* loss, float* mean, void* workspace,
                                    size_t workspace_bytes, void* stream);
/* Wait for the last tt_inbatch_softmax that used `workspace` (on `stream`)
 * and report TT_OK or TT_ERR_TIMEOUT. */
TT_API tt_status tt_inbatch_softmax_check(const void* workspace, void* stream);

/* Release a handle. Its work memory returns to a per-device pool that later
 * handles reuse (it is not returned to CUDA before the process exits); a
 * later user's stream first waits for the work this handle had enqueued, so
 * tt_free may be called while that work is still running. NULL is a no-op. */
TT_API void tt_free(tt_index* index);

/*
 * tt_score_topk_noalloc - tt_score_topk for callers that must not allocate
 * device memory while they run. (Not a step of the method: the pages have no
 * counterpart; it only changes where the work buffers live.)
 *
 * Who needs it: a process that reserved the GPU's memory up front (a serving
 * process with its own memory pool, where a late cudaMalloc fails or
 * fragments the pool), or a latency-bound loop in which cudaMalloc/cudaFree
 * would stall all work on the device. tt_score_topk keeps its buffers in the
 * index handle and grows them with cudaMalloc; this entry point calls no
 * allocator at all (no cudaMalloc, cudaFree, pinned host memory or handle):
 * its work buffers are one fixed array of TT_NOALLOC_SCRATCH_BYTES that the
 * library declares in device memory.
 *
 * Arguments: the corpus directly (rows: device [n, d] dtype; inv_norm:
 * device [n] f32 for a raw corpus, else NULL), then as tt_score_topk. Result,
 * exactness and asynchronous completion as tt_score_topk.
 *
 * Limits and rules:
 *   - b is limited by the array: about 128 KiB of work memory per query, so
 *     up to 255 queries per call; larger b is rejected with
 *     TT_ERR_UNSUPPORTED (tt_last_error() says how much was needed);
 *   - every call on a GPU uses the same array: calls that overlap on the GPU
 *     (two streams or two host threads at once) race and corrupt each other's
 *     results, so callers must serialise them;
 *   - the array keeps the previous call's contents; each call resets what it
 *     relies on before use;
 *   - when the array's memory is taken: CUDA loads a module's device memory
 *     when it is first used (lazy module loading, the default since CUDA
 *     12.2), so the 32 MiB of a GPU are committed by the first call on that
 *     GPU, which looks up the array's address with that GPU current; from then
 *     on it stays reserved until the process exits. Make one warm-up call per
 *     GPU at start-up, before any stream capture; later calls allocate nothing;
 *   - there is no handle to report a device-side timeout through: a search
 *     whose bounded wait expired leaves id -1 and score NaN in every output
 *     entry.
 */
#define TT_NOALLOC_SCRATCH_BYTES (32 * 1024 * 1024)

TT_API tt_status tt_score_topk_noalloc(const void* rows, tt_dtype dtype, int64_t n, int32_t d,
                                       const float* inv_norm, const void* queries, tt_dtype q_dtype,
                                       int32_t b, const uint32_t* exclude_bits, float tau, int32_t k,
                                       int32_t* out_ids, float* out_scores, void* stream);

/* Kernel-launch accounting and event timing (library-wide). Kinds: */
#define TT_KIND_NORMALIZE 0
#define TT_KIND_CAST 1
#define TT_KIND_STREAM 2
#define TT_KIND_TENSOR 3
#define TT_KIND_SELECT 4
#define TT_KIND_AUX 5
#define TT_KIND_SOFTMAX 6  /* tt_inbatch_softmax */
#define TT_KIND_ESTIMATE 7 /* the sampled threshold estimate of a small batch */
#define TT_NUM_KINDS 8

/* Total kernels this library has launched in the process. */
TT_API int64_t tt_launch_count(void);

/* Start recording a CUDA event pair around every subsequent launch, on the
 * launch stream. */
TT_API tt_status tt_profile_begin(void);

/* Stop recording, wait for the recorded events, and return per kind the
 * summed device time (ms) and the number of launches since tt_profile_begin.
 * Either array may be NULL; each has TT_NUM_KINDS entries. */
TT_API tt_status tt_profile_end(double* ms_per_kind, int64_t* launches_per_kind);

/* While recording (between tt_profile_begin and tt_profile_end): the launches
 * recorded so far, in order, as (kind, device ms), waiting for their events.
 * At most max_records are written; *n_records receives the number written. */
TT_API tt_status tt_profile_launches(int32_t* kinds, double* ms, int32_t max_records,
                                     int32_t* n_records);

/* Human-readable name of a status, and the last CUDA error text seen by the
 * calling thread (empty if none). */
TT_API const char* tt_status_string(tt_status status);
TT_API const char* tt_last_error(void);

/* Library version string. */
TT_API const char* tt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TT_H */
