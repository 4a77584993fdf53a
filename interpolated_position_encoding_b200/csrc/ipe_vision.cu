// Vision-tower kernels: position-table interpolation in merge order, the 2-D
// (row, col) rotary, their fused launch, and the plan read-back.
//
// "Qwen3-VL" notes (frankmowj.github.io), fast_pos_embed_interpolate,
// rot_pos_emb, apply_rotary_pos_emb_vision; cortiq-engine qwen3vis.rs
// (docs.rs), positions(), rope_angles(), attention().
#include "ipe_rotary_tma.cuh"

namespace ipe {

constexpr int kInterpThreads = 256;

// Channels of one interpolation block: 128 bytes of every output row.
template <typename T> constexpr int interp_slice() { return 128 / (int)sizeof(T); }

size_t interp_smem_bytes(bool bf16, int merge, int grid_side)
{
    const int cs = bf16 ? interp_slice<__nv_bfloat16>() : interp_slice<float>();
    return (size_t)merge * grid_side * cs * sizeof(float);
}

// ---------------------------------------------------------------- plan
template <int MAXIMG>
__global__ void vis_plan_kernel(const __grid_constant__ VisDesc<MAXIMG> d, int32_t *idx4, float *w4,
                                int32_t *rowcol)
{
    const long long N = d.n_patch;
    const int G = d.grid_side;
    for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < N;
         k += (long long)gridDim.x * blockDim.x) {
        const VisImage &im = d.img[find_image(d, k)];
        int row, col;
        patch_row_col(d, k, row, col);
        int y0, y1, x0, x1;
        float dy, dx;
        grid_sample(row, im.h, G, y0, y1, dy);
        grid_sample(col, im.w, G, x0, x1, dx);
        if (idx4) {
            idx4[0 * N + k] = y0 * G + x0;
            idx4[1 * N + k] = y0 * G + x1;
            idx4[2 * N + k] = y1 * G + x0;
            idx4[3 * N + k] = y1 * G + x1;
        }
        if (w4) {
            const float omdy = __fsub_rn(1.f, dy), omdx = __fsub_rn(1.f, dx);
            w4[0 * N + k] = __fmul_rn(omdy, omdx);
            w4[1 * N + k] = __fmul_rn(omdy, dx);
            w4[2 * N + k] = __fmul_rn(dy, omdx);
            w4[3 * N + k] = __fmul_rn(dy, dx);
        }
        if (rowcol) {
            rowcol[k] = row;
            rowcol[N + k] = col;
        }
    }
}

// -------------------------------------------------------- interpolation
// One block = one merge-row strip (m patch rows of one image, all w columns)
// x one 128-byte channel slice.  Bilinear interpolation is separable:
//   phase 1  R[iy][gx] = (1-dy) T[y0][gx] + dy T[y1][gx]   for the m rows, every
//            table column the strip samples (shared memory, fp32);
//   phase 2  out = (1-dx) R[iy][x0] + dx R[iy][x1], rounded once, written to
//            every frame (frames of a video repeat frame 0).
// Each table entry is read once per block instead of once per corner.
template <typename T, int MAXIMG>
__device__ __forceinline__ void interp_block(const VisDesc<MAXIMG> &d, const InterpArgs &ia, int strip,
                                             int slice, float4 *R)
{
    constexpr int CS = interp_slice<T>();
    constexpr int NV = CS / 4;                        // 4-channel vectors of a full slice
    const VisImage &im = d.img[find_image_of_strip(d, strip)];
    const int m = d.merge, G = d.grid_side, C = ia.hidden;
    const int by = strip - im.strip0;
    const int c0 = slice * CS;
    const int nv = min(CS, C - c0) / 4;
    int xl0, xl1;
    float dl;
    grid_sample(im.w - 1, im.w, G, xl0, xl1, dl);
    const int ncols = xl1 + 1;                        // columns 0 .. x1 of the last sample

    const T *tab = static_cast<const T *>(ia.table);
    for (int i = threadIdx.x; i < m * ncols * nv; i += blockDim.x) {
        const int v = i % nv;
        const int t2 = i / nv;
        const int gx = t2 % ncols, iy = t2 / ncols;
        int y0, y1;
        float dy;
        grid_sample(by * m + iy, im.h, G, y0, y1, dy);
        const float omdy = __fsub_rn(1.f, dy);
        const Pack<T, 4> a = ld_pack<T, 4>(tab + (size_t)(y0 * G + gx) * C + c0 + 4 * v);
        const Pack<T, 4> b = ld_pack<T, 4>(tab + (size_t)(y1 * G + gx) * C + c0 + 4 * v);
        float4 r;
        r.x = __fmaf_rn(dy, to_f32(b.v[0]), __fmul_rn(omdy, to_f32(a.v[0])));
        r.y = __fmaf_rn(dy, to_f32(b.v[1]), __fmul_rn(omdy, to_f32(a.v[1])));
        r.z = __fmaf_rn(dy, to_f32(b.v[2]), __fmul_rn(omdy, to_f32(a.v[2])));
        r.w = __fmaf_rn(dy, to_f32(b.v[3]), __fmul_rn(omdy, to_f32(a.v[3])));
        R[(iy * ncols + gx) * NV + v] = r;
    }
    __syncthreads();

    const long long hw = (long long)im.h * im.w;
    const long long strip_row0 = im.row0 + (long long)by * m * im.w;
    T *out = static_cast<T *>(ia.out);
    for (int i = threadIdx.x; i < m * im.w * nv; i += blockDim.x) {
        const int v = i % nv;
        const int p = i / nv;                         // patch of the strip, merge order
        const int bx = p / (m * m), rr = p - bx * m * m;
        const int iy = rr / m, ix = rr - iy * m;
        int x0, x1;
        float dx;
        grid_sample(bx * m + ix, im.w, G, x0, x1, dx);
        const float omdx = __fsub_rn(1.f, dx);
        const float4 r0 = R[(iy * ncols + x0) * NV + v];
        const float4 r1 = R[(iy * ncols + x1) * NV + v];
        Pack<T, 4> o;
        o.v[0] = from_f32<T>(__fmaf_rn(dx, r1.x, __fmul_rn(omdx, r0.x)));
        o.v[1] = from_f32<T>(__fmaf_rn(dx, r1.y, __fmul_rn(omdx, r0.y)));
        o.v[2] = from_f32<T>(__fmaf_rn(dx, r1.z, __fmul_rn(omdx, r0.z)));
        o.v[3] = from_f32<T>(__fmaf_rn(dx, r1.w, __fmul_rn(omdx, r0.w)));
        T *dst = out + (size_t)(strip_row0 + p) * C + c0 + 4 * v;
        for (int f = 0; f < im.t; ++f)
            st_pack<T, 4>(dst + (size_t)f * hw * C, o);
    }
}

template <typename T, int MAXIMG>
__global__ void __launch_bounds__(kInterpThreads) vis_interp_kernel(const __grid_constant__ VisDesc<MAXIMG> d,
                                                                    const __grid_constant__ InterpArgs ia)
{
    extern __shared__ float4 R[];
    const int b = blockIdx.x;
    interp_block<T, MAXIMG>(d, ia, b / ia.n_slices, b % ia.n_slices, R);
}

// --------------------------------------------------------------- fused
// Blocks [0, n_strips * n_slices) interpolate; the rest rotate q and k.
template <typename T, int VEC, int MAXIMG>
__global__ void __launch_bounds__(kRotThreads) vis_fused_kernel(const __grid_constant__ VisSrc<MAXIMG> src,
                                                                const __grid_constant__ InterpArgs ia,
                                                                const __grid_constant__ RotArgs r)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int n_interp = src.d.n_strips * ia.n_slices;
    if ((int)blockIdx.x < n_interp) {
        interp_block<T, MAXIMG>(src.d, ia, blockIdx.x / ia.n_slices, blockIdx.x % ia.n_slices,
                                reinterpret_cast<float4 *>(smem));
    } else {
        rotary_tiles<T, VEC, VisSrc<MAXIMG>>(r, src, blockIdx.x - n_interp, gridDim.x - n_interp, smem);
    }
}

// ------------------------------------------------------------- launches
template <int MAXIMG>
static VisDesc<MAXIMG> shrink(const VisDesc<1024> &d)
{
    VisDesc<MAXIMG> s;
    s.n_images = d.n_images;
    s.merge = d.merge;
    s.grid_side = d.grid_side;
    s.n_strips = d.n_strips;
    s.n_patch = d.n_patch;
    for (int i = 0; i < d.n_images && i < MAXIMG; ++i) s.img[i] = d.img[i];
    return s;
}

template <int MAXIMG>
static cudaError_t plan_impl(const VisDesc<1024> &d, int32_t *idx4, float *w4, int32_t *rowcol, cudaStream_t s)
{
    const long long blocks = std::min<long long>((d.n_patch + 255) / 256, (long long)sm_count() * 8);
    vis_plan_kernel<MAXIMG><<<(int)std::max<long long>(blocks, 1), 256, 0, s>>>(shrink<MAXIMG>(d), idx4, w4, rowcol);
    return cudaGetLastError();
}

cudaError_t launch_vis_plan(const VisDesc<1024> &d, int32_t *idx4, float *w4, int32_t *rowcol, cudaStream_t s)
{
    return d.n_images <= 16 ? plan_impl<16>(d, idx4, w4, rowcol, s) : plan_impl<1024>(d, idx4, w4, rowcol, s);
}

template <typename T, int MAXIMG>
static cudaError_t interp_impl(const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    const size_t smem = interp_smem_bytes(sizeof(T) == 2, d.merge, d.grid_side);
    auto kern = vis_interp_kernel<T, MAXIMG>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<d.n_strips * ia.n_slices, kInterpThreads, smem, s>>>(shrink<MAXIMG>(d), ia);
    return cudaGetLastError();
}

cudaError_t launch_vis_interp(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    if (bf16)
        return d.n_images <= 16 ? interp_impl<__nv_bfloat16, 16>(d, ia, s) : interp_impl<__nv_bfloat16, 1024>(d, ia, s);
    return d.n_images <= 16 ? interp_impl<float, 16>(d, ia, s) : interp_impl<float, 1024>(d, ia, s);
}

template <typename T, int MAXIMG>
static cudaError_t rope_impl(const VisDesc<1024> &d, const RotArgs &r, const VisAngleFreqs &f, cudaStream_t s)
{
    TmaRotArgs t;
    if (tma_rot_args(r, sizeof(T), t)) {
        t.aux_tma = 0;
        VisTmaSrc<MAXIMG> src{shrink<MAXIMG>(d), f};
        const int v = pick_vec(r, sizeof(T));
        if constexpr (sizeof(T) == 2) {
            if (v == 8) return launch_rotary_tma_vec<T, 8>(t, src, s);
        }
        if (v >= 4) return launch_rotary_tma_vec<T, 4>(t, src, s);
        return launch_rotary_tma_vec<T, 2>(t, src, s);   // VEC >= 2 on the TMA path
    }
    VisSrc<MAXIMG> src{shrink<MAXIMG>(d), f};
    return dispatch_vec<T>(r, src, s);
}

cudaError_t launch_vis_rope(bool bf16, const VisDesc<1024> &d, const RotArgs &r, const VisAngleFreqs &f,
                            cudaStream_t s)
{
    if (bf16)
        return d.n_images <= 16 ? rope_impl<__nv_bfloat16, 16>(d, r, f, s) : rope_impl<__nv_bfloat16, 1024>(d, r, f, s);
    return d.n_images <= 16 ? rope_impl<float, 16>(d, r, f, s) : rope_impl<float, 1024>(d, r, f, s);
}

template <typename T, int VEC, int MAXIMG>
static cudaError_t fused_vec(const VisDesc<1024> &d, const InterpArgs &ia, RotArgs r, const VisAngleFreqs &f,
                             cudaStream_t s)
{
    r.rows_per_tile = pick_rows_per_tile(r, VEC);
    const size_t smem = std::max(interp_smem_bytes(sizeof(T) == 2, d.merge, d.grid_side),
                                 rot_smem_bytes(r.rows_per_tile, r.half, false));
    auto kern = vis_fused_kernel<T, VEC, MAXIMG>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRotThreads, smem);
    if (e != cudaSuccess) return e;
    const long long ntiles = (r.rows + r.rows_per_tile - 1) / r.rows_per_tile;
    const long long n_rope = std::max<long long>(1, std::min(ntiles, (long long)sm_count() * std::max(per_sm, 1)));
    const long long n_interp = (long long)d.n_strips * ia.n_slices;
    VisSrc<MAXIMG> src{shrink<MAXIMG>(d), f};
    kern<<<(unsigned)(n_interp + n_rope), kRotThreads, smem, s>>>(src, ia, r);
    return cudaGetLastError();
}

template <typename T, int MAXIMG>
static cudaError_t fused_impl(const VisDesc<1024> &d, const InterpArgs &ia, const RotArgs &r,
                              const VisAngleFreqs &f, cudaStream_t s)
{
    const int v = pick_vec(r, sizeof(T));
    if constexpr (sizeof(T) == 2) {
        if (v == 8) return fused_vec<T, 8, MAXIMG>(d, ia, r, f, s);
    }
    if (v >= 4) return fused_vec<T, 4, MAXIMG>(d, ia, r, f, s);
    if (v == 2) return fused_vec<T, 2, MAXIMG>(d, ia, r, f, s);
    return fused_vec<T, 1, MAXIMG>(d, ia, r, f, s);
}

cudaError_t launch_vis_fused(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, const RotArgs &r,
                             const VisAngleFreqs &f, cudaStream_t s)
{
    if (bf16)
        return d.n_images <= 16 ? fused_impl<__nv_bfloat16, 16>(d, ia, r, f, s)
                                : fused_impl<__nv_bfloat16, 1024>(d, ia, r, f, s);
    return d.n_images <= 16 ? fused_impl<float, 16>(d, ia, r, f, s) : fused_impl<float, 1024>(d, ia, r, f, s);
}

}  // namespace ipe
