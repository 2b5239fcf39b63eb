// tt_rowdot.cuh - one row against one query with the streaming scorer's
// arithmetic, for the kernels that score rows one thread at a time outside
// the main passes (the small-batch threshold estimate and the exact
// fallback): an fp32 fused multiply-add chain over the row in element order
// (fp32 or bf16 rows against an fp32 query), or the exact int32 sum of code
// products (int8 rows against the query's packed codes).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tt.h"

namespace tt {

// The loads of a row are issued in batches of RB 16-byte pieces before the
// products that use them, so a row costs a few memory latencies, not one per
// piece; the products still run in element order.
constexpr int RB = 16;

__device__ __forceinline__ float dot_bf16(const __nv_bfloat16* row, const float* qf, int d) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
    float acc = 0.f;
    for (int i0 = 0; i0 < d / 8; i0 += RB) {
        uint4 r[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
            if (i0 + j < d / 8) r[j] = __ldcs(p + i0 + j);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            if (i0 + j >= d / 8) break;
            const uint32_t w[4] = {r[j].x, r[j].y, r[j].z, r[j].w};
            const float* q = qf + 8 * (i0 + j);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                acc = fmaf(__uint_as_float(w[t] << 16), q[2 * t], acc);
                acc = fmaf(__uint_as_float(w[t] & 0xFFFF0000u), q[2 * t + 1], acc);
            }
        }
    }
    return acc;
}

__device__ __forceinline__ float dot_f32(const float* row, const float* qf, int d) {
    const float4* p = reinterpret_cast<const float4*>(row);
    float acc = 0.f;
    for (int i0 = 0; i0 < d / 4; i0 += RB) {
        float4 r[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
            if (i0 + j < d / 4) r[j] = __ldcs(p + i0 + j);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            if (i0 + j >= d / 4) break;
            const float* q = qf + 4 * (i0 + j);
            acc = fmaf(r[j].x, q[0], acc);
            acc = fmaf(r[j].y, q[1], acc);
            acc = fmaf(r[j].z, q[2], acc);
            acc = fmaf(r[j].w, q[3], acc);
        }
    }
    return acc;
}

// d % 32 == 0
__device__ __forceinline__ int dot_i8(const int8_t* row, const int* qw, int d) {
    const int4* p = reinterpret_cast<const int4*>(row);
    int acc = 0;
    for (int i0 = 0; i0 < d / 16; i0 += RB) {
        int4 r[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
            if (i0 + j < d / 16) r[j] = __ldcs(p + i0 + j);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            if (i0 + j >= d / 16) break;
            const int* q = qw + 4 * (i0 + j);
            acc = __dp4a(r[j].x, q[0], acc);
            acc = __dp4a(r[j].y, q[1], acc);
            acc = __dp4a(r[j].z, q[2], acc);
            acc = __dp4a(r[j].w, q[3], acc);
        }
    }
    return acc;
}

// Stage query q for the dot products above: fp32 values (fp32 or bf16
// queries), or the packed int8 code words. Block-wide; the caller syncs.
__device__ __forceinline__ void stage_query(int dtype, const void* queries, int q_dtype, int q, int d, float* qf) {
    if (dtype == TT_I8) {
        const int* qw = reinterpret_cast<const int*>(queries) + (int64_t)q * (d / 4);
        for (int i = threadIdx.x; i < d / 4; i += blockDim.x) reinterpret_cast<int*>(qf)[i] = qw[i];
    } else {
        for (int i = threadIdx.x; i < d; i += blockDim.x) {
            const int64_t off = (int64_t)q * d + i;
            qf[i] = q_dtype == TT_F32 ? static_cast<const float*>(queries)[off]
                                      : __bfloat162float(static_cast<const __nv_bfloat16*>(queries)[off]);
        }
    }
}

// The score of row r: fl(dot * c_r) with c_r = fl(inv_norm_r * inv_tau)
// (inv_norm null: c = inv_tau); int8 rows: fl(fl(fl(acc) * us) * c_r) with
// c_r = fl(scale_r * inv_tau).
__device__ __forceinline__ float score_row(int dtype, const void* rows, int64_t r, int d, const float* qf,
                                           const float* inv_norm, float inv_tau, float us) {
    if (dtype == TT_I8) {
        const int acc = dot_i8(static_cast<const int8_t*>(rows) + r * d, reinterpret_cast<const int*>(qf), d);
        const float cj = inv_norm[r] * inv_tau;
        return (float)acc * us * cj;
    }
    const float acc = dtype == TT_F32 ? dot_f32(static_cast<const float*>(rows) + r * d, qf, d)
                                     : dot_bf16(static_cast<const __nv_bfloat16*>(rows) + r * d, qf, d);
    const float cj = inv_norm ? inv_norm[r] * inv_tau : inv_tau;
    return acc * cj;
}

}  // namespace tt
