// k_normalize.cu - K1: row-wise L2 normalisation of a corpus (or of a batch
// of queries), and the fp32 -> bf16 query cast.
//
// norm_j = sqrt(max(sum_i v_ji^2, 1e-12)), out_ji = v_ji / norm_j
// (x-algorithm recsys_two_tower_model.py, `_l2_normalize_candidates`; the
// user vector gets the same treatment in `RecsysTwoTowerModel.__call__`).
//
// HBM-bound: every row is read once with 16-byte loads and written once with
// 16-byte (or 8-byte) stores. L lanes of a warp share one row (L = 32 for
// rows of >= 512 bytes), each lane keeping up to 4 chunks in registers, and
// each warp works on two to four row groups at a time, with the loads of the
// next groups already issued, to keep enough bytes in flight. fp32 arithmetic with IEEE sqrt and division; the result is rounded
// to the output type to nearest-even.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_device.cuh"
#include "tt_internal.h"

namespace tt {
namespace {

constexpr int K1_THREADS = 256;

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int per_chunk = 4;
    __device__ static void unpack(const uint4& c, float* x) {
        x[0] = __uint_as_float(c.x);
        x[1] = __uint_as_float(c.y);
        x[2] = __uint_as_float(c.z);
        x[3] = __uint_as_float(c.w);
    }
};
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int per_chunk = 8;
    __device__ static void unpack(const uint4& c, float* x) {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

// Streaming 16-byte load (read once). Not the read-only path: `out` may
// alias `in`.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

// Store the normalised values of one input chunk (E elements) to out, at
// element offset `e0` of the row.
template <typename Tout, int E>
__device__ __forceinline__ void store_chunk(Tout* row_out, int e0, const float* y);

template <>
__device__ __forceinline__ void store_chunk<float, 4>(float* row_out, int e0, const float* y) {
    *reinterpret_cast<float4*>(row_out + e0) = make_float4(y[0], y[1], y[2], y[3]);
}
template <>
__device__ __forceinline__ void store_chunk<float, 8>(float* row_out, int e0, const float* y) {
    *reinterpret_cast<float4*>(row_out + e0) = make_float4(y[0], y[1], y[2], y[3]);
    *reinterpret_cast<float4*>(row_out + e0 + 4) = make_float4(y[4], y[5], y[6], y[7]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ void store_chunk<__nv_bfloat16, 4>(__nv_bfloat16* row_out, int e0,
                                                             const float* y) {
    *reinterpret_cast<uint2*>(row_out + e0) =
        make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
}
template <>
__device__ __forceinline__ void store_chunk<__nv_bfloat16, 8>(__nv_bfloat16* row_out, int e0,
                                                             const float* y) {
    *reinterpret_cast<uint4*>(row_out + e0) =
        make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                   pack_bf16x2(y[6], y[7]));
}

// Store E int8 codes at element offset e0 of the row; the code of element e
// is the low byte of qb[e] (two's complement).
__device__ __forceinline__ uint32_t pack_low_bytes(const uint32_t* qb) {
    const uint32_t lo = __byte_perm(qb[0], qb[1], 0x0040);  // bytes: qb0.b0, qb1.b0
    const uint32_t hi = __byte_perm(qb[2], qb[3], 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}
template <int E>
__device__ __forceinline__ void store_codes(int8_t* row_out, int e0, const uint32_t* qb);
template <>
__device__ __forceinline__ void store_codes<4>(int8_t* row_out, int e0, const uint32_t* qb) {
    *reinterpret_cast<uint32_t*>(row_out + e0) = pack_low_bytes(qb);
}
template <>
__device__ __forceinline__ void store_codes<8>(int8_t* row_out, int e0, const uint32_t* qb) {
    *reinterpret_cast<uint2*>(row_out + e0) = make_uint2(pack_low_bytes(qb), pack_low_bytes(qb + 4));
}

constexpr float K1_ROUND = 0x1.8p23f;

// The int8 coding quotient as the page writes it, fl(fl(v / norm) / scale)
// (norm == 0: v taken as given); the rare elements near a rounding boundary.
__device__ __noinline__ float ieee_code_quotient(float v, float norm, float scale) {
    const float w = norm != 0.0f ? __fdiv_rn(v, norm) : v;
    return __fdiv_rn(w, scale);
}

// MODE 0: out rows = v / norm (Tout). MODE 1: inv_norm[j] = 1 / norm.
// MODE 2: w = v / norm, then int8 codes of w to out (Tout = int8_t) and the
// row's scale to inv_norm. MODE 3: the same coding of v as given (queries).
// L lanes per row, CPL 16-byte chunks per lane (d * elem <= 2048 bytes),
// U row groups per warp in flight at once.
template <typename Tin, typename Tout, int MODE, int L, int CPL, int U>
__global__ void __launch_bounds__(K1_THREADS)
    k1_normalize(const Tin* in, int64_t n, int d, Tout* out,
                 float* __restrict__ inv_norm) {
    constexpr int E = Elem<Tin>::per_chunk;
    constexpr int ROWS_PER_GROUP = 32 / L;
    const int chunks = d / E;
    const int lane = threadIdx.x & 31;
    const int sub = lane % L;
    const int grp = lane / L;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t step = nwarps * (U * ROWS_PER_GROUP);

    // The loads of the next row groups are issued before the current ones
    // are reduced, so each warp keeps two groups of loads in flight.
    auto load_group = [&](int64_t gbase, uint4 (&dst)[U][CPL]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = gbase + u * ROWS_PER_GROUP + grp;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = sub + i * L;
                if (r < n && c < chunks)
                    dst[u][i] = ld_stream(in + r * d + (int64_t)c * E);
                else
                    dst[u][i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // (Rows of 512 bytes and more, where the doubled registers fit: up to 4
    // chunks per lane and group.)
    constexpr bool PREFETCH = L == 32 && U * CPL <= 4;
    uint4 nxt[U][CPL];
    int64_t base = warp * (U * ROWS_PER_GROUP);
    if (PREFETCH && base < n) load_group(base, nxt);
    for (; base < n; base += step) {
        int64_t row[U];
#pragma unroll
        for (int u = 0; u < U; ++u) row[u] = base + u * ROWS_PER_GROUP + grp;
        uint4 raw[U][CPL];
        if (PREFETCH) {
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < CPL; ++i) raw[u][i] = nxt[u][i];
            if (base + step < n) load_group(base + step, nxt);
        } else {
            load_group(base, raw);
        }
        float ss[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            ss[u] = 0.f;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                float x[E];
                Elem<Tin>::unpack(raw[u][i], x);
#pragma unroll
                for (int e = 0; e < E; ++e) ss[u] = fmaf(x[e], x[e], ss[u]);
            }
        }
#pragma unroll
        for (int off = L / 2; off > 0; off >>= 1) {
#pragma unroll
            for (int u = 0; u < U; ++u) ss[u] += __shfl_xor_sync(0xFFFFFFFFu, ss[u], off);
        }
        if constexpr (MODE >= 2) {
            // int8 coding (recsys_two_tower_model.py `compute_top_k_int8`):
            // w = fl(v / norm) (MODE 2; MODE 3: w = v), scale = max(fl(max|w|
            // / 127), 1e-12), code = clip(round_half_even(fl(w / scale))),
            // every step an IEEE fp32 operation as written there. Two
            // divisions per element are not needed for that result:
            //  - dividing by a positive norm is monotone, so max|w| =
            //    fl(max|v| / norm): one division per row gives the scale;
            //  - y = fl(fl(v * fl(1/norm)) * fl(1/scale)) differs from the
            //    IEEE quotient fl(w / scale) by at most four relative
            //    roundings, |y| * 2^-21 in all, so round(y) is the exact code
            //    unless y lies within that distance of a half-integer; such
            //    rare elements (the margin below is four times wider) take
            //    the two IEEE divisions.
            float mv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                mv[u] = 0.f;
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    float x[E];
                    Elem<Tin>::unpack(raw[u][i], x);
#pragma unroll
                    for (int e = 0; e < E; ++e) mv[u] = fmaxf(mv[u], fabsf(x[e]));
                }
            }
#pragma unroll
            for (int off = L / 2; off > 0; off >>= 1) {
#pragma unroll
                for (int u = 0; u < U; ++u) mv[u] = fmaxf(mv[u], __shfl_xor_sync(0xFFFFFFFFu, mv[u], off));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (row[u] >= n) continue;
                const float norm = MODE == 2 ? __fsqrt_rn(fmaxf(ss[u], 1e-12f)) : 1.0f;
                const float mx = MODE == 2 ? __fdiv_rn(mv[u], norm) : mv[u];  // max_i |fl(v_i / norm)|
                const float scale = fmaxf(__fdiv_rn(mx, 127.0f), 1e-12f);
                const float rn = MODE == 2 ? __frcp_rn(norm) : 1.0f;
                const float rs = __frcp_rn(scale);
                if (sub == 0) inv_norm[row[u]] = scale;
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    const int c = sub + i * L;
                    if (c < chunks) {
                        float x[E];
                        Elem<Tin>::unpack(raw[u][i], x);
                        uint32_t qb[E];
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            float y = (MODE == 2 ? x[e] * rn : x[e]) * rs;
                            // Adding 1.5 * 2^23 rounds y to an integer, ties to
                            // even, and leaves it in the low mantissa bits of t
                            // (|y| < 2^22); subtracting it back gives rint(y).
                            float t = __fadd_rn(y, K1_ROUND);
                            const float to_int = fabsf(__fadd_rn(y, -__fadd_rn(t, -K1_ROUND)));
                            if (!(0.5f - to_int > fabsf(y) * 0x1p-19f + 0x1p-19f)) {
                                y = ieee_code_quotient(x[e], MODE == 2 ? norm : 0.0f, scale);
                                t = __fadd_rn(y, K1_ROUND);
                            }
                            // |y| <= 127 (1 + 2^-20) < 127.5 because scale >=
                            // max|w| / 127 up to one rounding, so the page's clip
                            // to [-127, 127] never changes a code; the low byte
                            // of t is the code in two's complement.
                            qb[e] = __float_as_uint(t);
                        }
                        store_codes<E>(reinterpret_cast<int8_t*>(out) + row[u] * d, c * E, qb);
                    }
                }
            }
        } else {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (row[u] >= n) continue;
                const float norm = __fsqrt_rn(fmaxf(ss[u], 1e-12f));
                if constexpr (MODE == 1) {
                    if (sub == 0) inv_norm[row[u]] = __fdiv_rn(1.0f, norm);
                } else {
#pragma unroll
                    for (int i = 0; i < CPL; ++i) {
                        const int c = sub + i * L;
                        if (c < chunks) {
                            float x[E], y[E];
                            Elem<Tin>::unpack(raw[u][i], x);
#pragma unroll
                            for (int e = 0; e < E; ++e) y[e] = __fdiv_rn(x[e], norm);
                            store_chunk<Tout, E>(out + row[u] * d, c * E, y);
                        }
                    }
                }
            }
        }
    }
}

__global__ void k0_cast_bf16(const float4* __restrict__ in, int64_t count4, uint2* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = in[i];
        out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

template <typename Tin, typename Tout, int MODE>
cudaError_t dispatch_lanes(const void* in, int64_t n, int d, void* out, cudaStream_t s, void* aux = nullptr) {
    constexpr int E = Elem<Tin>::per_chunk;
    const int chunks = d / E;
    int L = 32;
    while (L > chunks) L >>= 1;
    if (MODE >= 2) {
        // int8 coding does per-row work (a square root, two divisions, two
        // reciprocals, two reductions) that every lane of a row repeats:
        // fewer lanes per row (up to four chunks each) spread it over
        // several rows at once. (32 lanes per 512-byte row ran at 0.41 of
        // HBM; plain normalisation, with less per-row work, at 0.94.)
        L = 4;
        while (L < 32 && L * 4 < chunks) L <<= 1;
    }
    const int cpl = (chunks + L - 1) / L;
    const int unroll = (L == 32 && cpl == 1) ? 4 : 2;
    const int rows_per_block = (K1_THREADS / 32) * unroll * (32 / L);
    int64_t blocks = (n + rows_per_block - 1) / rows_per_block;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t max_blocks = (int64_t)sms * (2048 / K1_THREADS);
    if (blocks > max_blocks) blocks = max_blocks;
    if (blocks < 1) blocks = 1;
    const Tin* pin = static_cast<const Tin*>(in);
    Tout* pout = (MODE == 0 || MODE >= 2) ? static_cast<Tout*>(out) : nullptr;
    float* pinv = MODE == 1 ? static_cast<float*>(out) : static_cast<float*>(aux);
    note_launch_begin(TT_KIND_NORMALIZE, s);
    const dim3 g((unsigned)blocks), t(K1_THREADS);
    if (MODE >= 2) {
        if (L == 4) k1_normalize<Tin, Tout, MODE, 4, 4, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
        else if (L == 8) k1_normalize<Tin, Tout, MODE, 8, 4, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
        else if (L == 16) k1_normalize<Tin, Tout, MODE, 16, 4, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
        else k1_normalize<Tin, Tout, MODE, 32, 4, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    } else if (L == 32 && cpl == 1) k1_normalize<Tin, Tout, MODE, 32, 1, 4><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else if (L == 32 && cpl == 2) k1_normalize<Tin, Tout, MODE, 32, 2, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else if (L == 32) k1_normalize<Tin, Tout, MODE, 32, 4, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else if (L == 16) k1_normalize<Tin, Tout, MODE, 16, 2, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else if (L == 8) k1_normalize<Tin, Tout, MODE, 8, 2, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else if (L == 4) k1_normalize<Tin, Tout, MODE, 4, 2, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    else k1_normalize<Tin, Tout, MODE, 2, 2, 2><<<g, t, 0, s>>>(pin, n, d, pout, pinv);
    note_launch_end(TT_KIND_NORMALIZE, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_normalize(const void* in, int in_dtype, int64_t n, int d, void* out,
                             int out_dtype, int mode, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    if (in_dtype == TT_F32) {
        if (mode == TT_NORM_FUSED) return dispatch_lanes<float, float, 1>(in, n, d, out, s);
        if (out_dtype == TT_F32) return dispatch_lanes<float, float, 0>(in, n, d, out, s);
        return dispatch_lanes<float, __nv_bfloat16, 0>(in, n, d, out, s);
    }
    if (mode == TT_NORM_FUSED) return dispatch_lanes<__nv_bfloat16, float, 1>(in, n, d, out, s);
    if (out_dtype == TT_F32) return dispatch_lanes<__nv_bfloat16, float, 0>(in, n, d, out, s);
    return dispatch_lanes<__nv_bfloat16, __nv_bfloat16, 0>(in, n, d, out, s);
}

cudaError_t launch_quantize(const void* in, int in_dtype, int64_t n, int d, int8_t* codes, float* scales,
                            bool normalise, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    if (in_dtype == TT_F32)
        return normalise ? dispatch_lanes<float, int8_t, 2>(in, n, d, codes, s, scales)
                         : dispatch_lanes<float, int8_t, 3>(in, n, d, codes, s, scales);
    return normalise ? dispatch_lanes<__nv_bfloat16, int8_t, 2>(in, n, d, codes, s, scales)
                     : dispatch_lanes<__nv_bfloat16, int8_t, 3>(in, n, d, codes, s, scales);
}

cudaError_t launch_cast_bf16(const float* in, int64_t count, __nv_bfloat16* out, cudaStream_t s) {
    const int64_t count4 = count / 4;  // count is a multiple of 16 (d % 16 == 0)
    if (count4 == 0) return cudaSuccess;
    int64_t blocks = (count4 + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    note_launch_begin(TT_KIND_CAST, s);
    k0_cast_bf16<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(in), count4,
                                                  reinterpret_cast<uint2*>(out));
    note_launch_end(TT_KIND_CAST, s);
    return cudaGetLastError();
}

}  // namespace tt
