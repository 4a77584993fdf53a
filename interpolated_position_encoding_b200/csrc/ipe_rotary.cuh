// In-place rotation engine shared by the text MRoPE and vision 2-D rotary
// kernels.
//
// Rows (tokens or patches) are processed in tiles of `rows_per_tile`.  For a
// tile the block first fills shared memory with one (cos, sin) pair per
// (row, frequency) -- computed once, shared by every head of q and k -- and
// then streams the rotary channels of all head rows through registers with
// vector loads and stores (`VEC` elements per access), several accesses in
// flight per thread.
#pragma once

#include <algorithm>

#include "ipe_device.cuh"

namespace ipe {

constexpr int kRotThreads = 256;
constexpr int kRotBatch = 4;       // independent head-row chunks in flight per thread

// ------------------------------------------------------------ angle sources
// prepare(): write lo[pr * half + j] = (cos, sin) of frequency j of tile row
// pr (and hi[...] for the second half when kHi); must end with the block
// having written everything (the caller synchronises afterwards).

struct MropeSrc {
    static constexpr bool kHi = false;
    static constexpr bool kHf = false;
    MropeAngles a;
    __device__ __forceinline__ void prepare(long long r0, int rows, int half, float2 *lo, float2 *,
                                            int *) const
    {
        for (int i = threadIdx.x; i < rows * half; i += blockDim.x) {
            const int pr = i / half, j = i - pr * half;
            const int ax = mrope_axis(j, a.section, a.interleaved);
            const int pos = __ldg(a.positions + (long long)ax * a.T + r0 + pr);
            // fl32(fl32(pos) * inv_freq[j]): one rounded product, no contraction
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            float s, c;
            sincosf(angle, &s, &c);
            lo[i] = make_float2(c, s);
        }
    }
};

struct TableSrc {
    static constexpr bool kHi = true;
    static constexpr bool kHf = false;
    TableAngles a;
    __device__ __forceinline__ void prepare(long long r0, int rows, int half, float2 *lo, float2 *hi,
                                            int *) const
    {
        const int rot = 2 * half;
        for (int i = threadIdx.x; i < rows * half; i += blockDim.x) {
            const int pr = i / half, j = i - pr * half;
            const long long o = (r0 + pr) * rot + j;
            lo[i] = make_float2(__ldg(a.cos + o), __ldg(a.sin + o));
            hi[i] = make_float2(__ldg(a.cos + o + half), __ldg(a.sin + o + half));
        }
    }
};

template <int MAXIMG>
struct VisSrc {
    static constexpr bool kHi = false;
    static constexpr bool kHf = false;
    VisDesc<MAXIMG> d;
    VisAngleFreqs f;
    // aux: (row, col) of each tile row.
    __device__ __forceinline__ void prepare(long long r0, int rows, int half, float2 *lo, float2 *,
                                            int *aux) const
    {
        for (int pr = threadIdx.x; pr < rows; pr += blockDim.x) {
            int row, col;
            patch_row_col(d, r0 + pr, row, col);
            aux[2 * pr] = row;
            aux[2 * pr + 1] = col;
        }
        __syncthreads();
        const int nf = f.nf;
        for (int i = threadIdx.x; i < rows * half; i += blockDim.x) {
            const int pr = i / half, j = i - pr * half;
            // angles [row * inv (nf) | col * inv (nf)]
            const int axis = j < nf ? 0 : 1;
            const int fi = j < nf ? j : j - nf;
            const float angle = __fmul_rn(__int2float_rn(aux[2 * pr + axis]), f.inv[fi]);
            float s, c;
            sincosf(angle, &s, &c);
            lo[i] = make_float2(c, s);
        }
    }
};

// HF rounding mode of a source: cos / sin cast to the activation dtype T
// (each thread rounds the entries it wrote in prepare()).
template <class Base, typename T>
struct HfVecSrc : Base {
    static constexpr bool kHf = true;
    __device__ __forceinline__ void prepare(long long r0, int rows, int half, float2 *lo, float2 *hi, int *aux) const
    {
        Base::prepare(r0, rows, half, lo, hi, aux);
        for (int i = threadIdx.x; i < rows * half; i += blockDim.x) {
            lo[i] = make_float2(round_to_dtype<T>(lo[i].x), round_to_dtype<T>(lo[i].y));
            if constexpr (Base::kHi) hi[i] = make_float2(round_to_dtype<T>(hi[i].x), round_to_dtype<T>(hi[i].y));
        }
    }
};

// Shared-memory bytes of one rotation block.
__host__ __device__ inline size_t rot_smem_bytes(int rows_per_tile, int half, bool hi)
{
    return (size_t)rows_per_tile * half * sizeof(float2) * (hi ? 2 : 1) +
           (size_t)rows_per_tile * 2 * sizeof(int);
}

// Process tiles bid, bid + nb, ... of the rows of `r`.
template <typename T, int VEC, class Src>
__device__ __forceinline__ void rotary_tiles(const RotArgs &r, const Src &src, long long bid, long long nb,
                                             unsigned char *smem)
{
    const int half = r.half;
    const int rpt = r.rows_per_tile;
    float2 *lo = reinterpret_cast<float2 *>(smem);
    float2 *hi = Src::kHi ? lo + (size_t)rpt * half : lo;
    int *aux = reinterpret_cast<int *>(lo + (size_t)rpt * half * (Src::kHi ? 2 : 1));

    const int heads = r.hq + r.hk;
    const int nvec = half / VEC;
    const int per_row = heads * nvec;
    const long long ntiles = (r.rows + rpt - 1) / rpt;
    T *const q = static_cast<T *>(r.q);
    T *const k = static_cast<T *>(r.k);

    for (long long tile = bid; tile < ntiles; tile += nb) {
        const long long r0 = tile * rpt;
        const int rows = (int)min((long long)rpt, r.rows - r0);
        src.prepare(r0, rows, half, lo, hi, aux);
        __syncthreads();

        const int tasks = rows * per_row;
        for (int base = threadIdx.x; base < tasks; base += blockDim.x * kRotBatch) {
            T *ptr[kRotBatch];
            int cs[kRotBatch];
            Pack<T, VEC> xa[kRotBatch], xb[kRotBatch];
#pragma unroll
            for (int b = 0; b < kRotBatch; ++b) {
                const int i = base + b * blockDim.x;
                ptr[b] = nullptr;
                if (i < tasks) {
                    const int u = i % nvec;
                    const int t2 = i / nvec;
                    const int h = t2 % heads;
                    const int pr = t2 / heads;
                    const long long row = r0 + pr;
                    T *p = h < r.hq ? q + row * r.q_stride + (long long)h * r.head_dim
                                    : k + row * r.k_stride + (long long)(h - r.hq) * r.head_dim;
                    ptr[b] = p + u * VEC;
                    cs[b] = pr * half + u * VEC;
                    xa[b] = ld_pack<T, VEC>(ptr[b]);
                    xb[b] = ld_pack<T, VEC>(ptr[b] + half);
                }
            }
#pragma unroll
            for (int b = 0; b < kRotBatch; ++b) {
                if (ptr[b] == nullptr) continue;
                Pack<T, VEC> ya, yb;
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float2 cl = lo[cs[b] + e];
                    const float2 ch = Src::kHi ? hi[cs[b] + e] : cl;
                    const float a = to_f32(xa[b].v[e]);
                    const float bb = to_f32(xb[b].v[e]);
                    // x[j] cos - x[j+h] sin ; x[j+h] cos + x[j] sin
                    if constexpr (Src::kHf) {
                        // each product rounded to T, the sum in fp32, then to T
                        ya.v[e] = from_f32<T>(__fadd_rn(round_to_dtype<T>(__fmul_rn(a, cl.x)),
                                                        round_to_dtype<T>(-__fmul_rn(bb, cl.y))));
                        yb.v[e] = from_f32<T>(__fadd_rn(round_to_dtype<T>(__fmul_rn(bb, ch.x)),
                                                        round_to_dtype<T>(__fmul_rn(a, ch.y))));
                    } else {
                        ya.v[e] = from_f32<T>(__fmaf_rn(a, cl.x, -__fmul_rn(bb, cl.y)));
                        yb.v[e] = from_f32<T>(__fmaf_rn(bb, ch.x, __fmul_rn(a, ch.y)));
                    }
                }
                st_pack<T, VEC>(ptr[b], ya);
                st_pack<T, VEC>(ptr[b] + half, yb);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- launch
inline int sm_count()
{
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// ------------------------------------------------------------- rotation
template <typename T, int VEC, class Src>
__global__ void __launch_bounds__(kRotThreads) rotary_kernel(const __grid_constant__ RotArgs r,
                                                             const __grid_constant__ Src src)
{
    extern __shared__ __align__(16) unsigned char smem[];
    rotary_tiles<T, VEC, Src>(r, src, blockIdx.x, gridDim.x, smem);
}

// Rows per tile: about 2048 head-row chunks per tile, at most 64 rows.
inline int pick_rows_per_tile(const RotArgs &r, int vec)
{
    const int per_row = (r.hq + r.hk) * (r.half / vec);
    int rpt = 2048 / std::max(per_row, 1);
    return std::max(1, std::min(rpt, 64));
}

template <typename T, int VEC, class Src>
cudaError_t launch_rotary_vec(RotArgs r, const Src &src, cudaStream_t s)
{
    r.rows_per_tile = pick_rows_per_tile(r, VEC);
    const size_t smem = rot_smem_bytes(r.rows_per_tile, r.half, Src::kHi);
    auto kern = rotary_kernel<T, VEC, Src>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRotThreads, smem);
    if (e != cudaSuccess) return e;
    const long long ntiles = (r.rows + r.rows_per_tile - 1) / r.rows_per_tile;
    const long long cap = (long long)sm_count() * std::max(per_sm, 1);
    const int blocks = (int)std::max<long long>(1, std::min(ntiles, cap));
    kern<<<blocks, kRotThreads, smem, s>>>(r, src);
    return cudaGetLastError();
}

template <typename T, class Src>
cudaError_t dispatch_vec(const RotArgs &r, const Src &src, cudaStream_t s)
{
    const int v = pick_vec(r, sizeof(T));
    if constexpr (sizeof(T) == 2) {
        if (v == 8) return launch_rotary_vec<T, 8, Src>(r, src, s);
    }
    if (v >= 4) return launch_rotary_vec<T, 4, Src>(r, src, s);
    if (v == 2) return launch_rotary_vec<T, 2, Src>(r, src, s);
    return launch_rotary_vec<T, 1, Src>(r, src, s);
}


}  // namespace ipe
