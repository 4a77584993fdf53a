// Device helpers shared by the kernels: element conversion, vector packs, the
// vision index decode and the multimodal axis rule.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ipe_internal.h"

namespace ipe {

// ----------------------------------------------------------- element types
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// Packed bf16 arithmetic with one rounding per result.  For bf16 operands
// these equal the fp32 operation followed by rounding to bf16:
//   * the exact product of two bf16 values (8-bit significands) fits in fp32;
//   * an fp32 sum of two bf16 values is inexact only when their exponents
//     differ by 16 or more.  The sum then lies within 2^(e-15) of the larger
//     operand a (exponent e), while the nearest bf16 rounding midpoints are
//     at least 2^(e-9) from a, so both roundings give a.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// v rounded to the dtype T and back to fp32 (round to nearest even; exact for fp32).
template <typename T> __device__ __forceinline__ float round_to_dtype(float v) { return to_f32(from_f32<T>(v)); }

// N contiguous elements moved as one aligned access (N * sizeof(T) <= 16).
template <typename T, int N>
struct __align__(sizeof(T) * N) Pack {
    T v[N];
};

template <typename T, int N>
__device__ __forceinline__ Pack<T, N> ld_pack(const T *p)
{
    return *reinterpret_cast<const Pack<T, N> *>(p);
}

template <typename T, int N>
__device__ __forceinline__ void st_pack(T *p, const Pack<T, N> &v)
{
    *reinterpret_cast<Pack<T, N> *>(p) = v;
}

// ------------------------------------------------------ multimodal axis rule
// Axis (0 = T, 1 = H, 2 = W) that frequency j follows.
// Interleaved ("M01 RMSNorm and multimodal RoPE", problem summary): H if
// j % 3 == 1 and j < 3 s_h, W if j % 3 == 2 and j < 3 s_w, otherwise T.
// Chunked (same page, layout table): T below s_t, H below s_t + s_h, then W.
__device__ __forceinline__ int mrope_axis(int j, const int *section, int interleaved)
{
    if (interleaved) {
        const int r = j % 3;
        if (r == 1 && j < 3 * section[1]) return 1;
        if (r == 2 && j < 3 * section[2]) return 2;
        return 0;
    }
    if (j < section[0]) return 0;
    if (j < section[0] + section[1]) return 1;
    return 2;
}

// --------------------------------------------------------- vision indexing
// Image holding global patch k (largest i with row0 <= k).
template <int MAXIMG>
__device__ __forceinline__ int find_image(const VisDesc<MAXIMG> &d, long long k)
{
    int lo = 0, hi = d.n_images - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (d.img[mid].row0 <= k) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Image holding merge-row strip s.
template <int MAXIMG>
__device__ __forceinline__ int find_image_of_strip(const VisDesc<MAXIMG> &d, int s)
{
    int lo = 0, hi = d.n_images - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (d.img[mid].strip0 <= s) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// (row, col) of patch k on its image's grid.  Output order within an image:
// frame, merge-block row, merge-block column, then the m x m block row-major
// ("Qwen3-VL" notes, fast_pos_embed_interpolate and rot_pos_emb).
template <int MAXIMG>
__device__ __forceinline__ void patch_row_col(const VisDesc<MAXIMG> &d, long long k, int &row, int &col)
{
    const VisImage &im = d.img[find_image(d, k)];
    const int m = d.merge;
    // 32-bit from here: a request holds fewer than 2^31 patches (the host
    // checks), so the patch's offset in its image and h * w fit in an int
    const int hw = im.h * im.w;
    const int q = (int)(k - im.row0) % hw;         // index within the frame
    int blk, iy, ix;                                // merge block, row and column inside it
    if (m == 2) {
        blk = q >> 2;
        iy = (q >> 1) & 1;
        ix = q & 1;
    } else {
        blk = q / (m * m);
        const int r = q - blk * m * m;
        iy = r / m;
        ix = r - iy * m;
    }
    const int wb = im.w / m;
    const int by = blk / wb, bx = blk - by * wb;
    row = by * m + iy;
    col = bx * m + ix;
}

// Sample point i of n on a grid of side G: floor index i0, clipped ceiling
// i1 and fraction d of i (G-1) / (n-1) (0 when n == 1).  Integer quotient and
// remainder make i0 exact; d is the correctly rounded fp32 quotient.
__device__ __forceinline__ void grid_sample(int i, int n, int G, int &i0, int &i1, float &d)
{
    if (n == 1) {
        i0 = 0;
        d = 0.f;
    } else {
        const int num = i * (G - 1);
        i0 = num / (n - 1);
        const int rem = num - i0 * (n - 1);
        d = __fdiv_rn((float)rem, (float)(n - 1));
    }
    i1 = min(i0 + 1, G - 1);
}

}  // namespace ipe
