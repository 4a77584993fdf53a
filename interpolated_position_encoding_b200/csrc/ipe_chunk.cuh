// Head rows held as 16-byte chunks, one chunk per lane: the shared arithmetic
// of the fused QK-RMSNorm + rotary kernels (prefill and decode).
//
// A head row of D elements is spread over LPR = D / EC lanes (EC = 8 bf16 or
// 4 fp32 elements per 16-byte chunk).  The row's sum of squares is reduced
// with shuffles inside those LPR lanes, and the rotary partner of a chunk
// (the chunk half a rotary slice away) is fetched from its lane by shuffle.
#pragma once

#include "ipe_rotary_tma.cuh"

namespace ipe {

template <typename T> struct QkElem;
template <> struct QkElem<__nv_bfloat16> {
    static constexpr int EC = 8;
};
template <> struct QkElem<float> {
    static constexpr int EC = 4;
};

// A 16-byte chunk (4 words) as EC/2 fp32 pairs, and back (one rounding to
// the dtype per element).
template <typename T> __device__ __forceinline__ void chunk_to_pairs(const uint32_t *w, float2 *p);
template <> __device__ __forceinline__ void chunk_to_pairs<__nv_bfloat16>(const uint32_t *w, float2 *p)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}
template <> __device__ __forceinline__ void chunk_to_pairs<float>(const uint32_t *w, float2 *p)
{
#pragma unroll
    for (int i = 0; i < 2; ++i) p[i] = make_float2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
}
template <typename T> __device__ __forceinline__ void pairs_to_chunk(const float2 *p, uint32_t *w);
template <> __device__ __forceinline__ void pairs_to_chunk<__nv_bfloat16>(const float2 *p, uint32_t *w)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(p[i].x, p[i].y);
        w[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
}
template <> __device__ __forceinline__ void pairs_to_chunk<float>(const float2 *p, uint32_t *w)
{
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        w[2 * i] = __float_as_uint(p[i].x);
        w[2 * i + 1] = __float_as_uint(p[i].y);
    }
}

// RMSNorm of the row whose chunk x this lane holds: y = dtype(dtype(x r) * w)
// with r = rsqrt(mean(x^2) + eps) in fp32 (inv_d = 1 / D, exact: D is a power
// of two).  Every lane of the warp must call it (shuffles over LPR lanes).
template <typename T, int LPR>
__device__ __forceinline__ Pack<uint32_t, 4> rms_norm_chunk(const Pack<uint32_t, 4> &x, const uint32_t *w, float inv_d,
                                                            float eps)
{
    constexpr int NP = QkElem<T>::EC / 2;
    float2 xv[NP];
    chunk_to_pairs<T>(x.v, xv);
    float2 acc = mul2(xv[0], xv[0]);
#pragma unroll
    for (int i = 1; i < NP; ++i) acc = fma2(xv[i], xv[i], acc);
    float ss = __fadd_rn(acc.x, acc.y);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, LPR);
    const float r = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, inv_d), eps));
    // cast back first, then the weight
    const float2 r2 = make_float2(r, r);
#pragma unroll
    for (int i = 0; i < NP; ++i) xv[i] = mul2(xv[i], r2);
    Pack<uint32_t, 4> y;
    pairs_to_chunk<T>(xv, y.v);
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
        for (int i = 0; i < 4; ++i) y.v[i] = mul_bf16x2(y.v[i], w[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) y.v[i] = __float_as_uint(__fmul_rn(__uint_as_float(y.v[i]), __uint_as_float(w[i])));
    }
    return y;
}

// Rotation of the chunk y by the pairs (co, si), si carrying the sign of the
// chunk's half (-sin on the first half, +sin on the second; pass-through
// chunks: co 1, si 0): out = y cos + partner(y) si.  Every lane of the warp
// must call it (one shuffle per word).
template <typename T>
__device__ __forceinline__ Pack<uint32_t, 4> rotate_row_chunk(const Pack<uint32_t, 4> &y, const float2 *co, const float2 *si,
                                                          int partner)
{
    constexpr int NP = QkElem<T>::EC / 2;
    Pack<uint32_t, 4> yp;
#pragma unroll
    for (int i = 0; i < 4; ++i) yp.v[i] = __shfl_sync(0xffffffffu, y.v[i], partner);
    float2 yv[NP], pv[NP];
    chunk_to_pairs<T>(y.v, yv);
    chunk_to_pairs<T>(yp.v, pv);
#pragma unroll
    for (int i = 0; i < NP; ++i) yv[i] = fma2(yv[i], co[i], mul2(pv[i], si[i]));
    Pack<uint32_t, 4> o;
    pairs_to_chunk<T>(yv, o.v);
    return o;
}

}  // namespace ipe
