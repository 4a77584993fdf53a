// Vision-tower kernels: position-table interpolation in merge order, the 2-D
// (row, col) rotary, and the plan read-back.
//
// "Qwen3-VL" notes (frankmowj.github.io), fast_pos_embed_interpolate,
// rot_pos_emb, apply_rotary_pos_emb_vision; cortiq-engine qwen3vis.rs
// (docs.rs), positions(), rope_angles(), attention().
#include "ipe_rotary_tma.cuh"

namespace ipe {

constexpr int kInterpThreads = 256;

// Channels of one interpolation block: 128 bytes of every output row.
template <typename T> constexpr int interp_slice() { return 128 / (int)sizeof(T); }

// Column samples cached per block (images at most this wide; wider ones
// recompute each sample).  512 keeps four two-slice blocks on an SM.
constexpr int kColCache = 512;

size_t interp_smem_bytes(bool bf16, int merge, int grid_side, int slices)
{
    const int cs = bf16 ? interp_slice<__nv_bfloat16>() : interp_slice<float>();
    return (size_t)merge * grid_side * slices * cs * sizeof(float) + (kColCache + merge) * sizeof(int2);
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
// x U consecutive 128-byte channel slices.  Bilinear interpolation is
// separable:
//   phase 1  R[iy][gx] = (1-dy) T[y0][gx] + dy T[y1][gx]   for the m rows, every
//            table column the strip samples (shared memory, fp32);
//   phase 2  out = (1-dx) R[iy][x0] + dx R[iy][x1], rounded once, written to
//            every frame (frames of a video repeat frame 0).
// Each table entry is read once per block instead of once per corner.  Lane
// v of a row moves chunk v of each of the U slices (E channels, 16 bytes
// when rows are 16-byte aligned), so the block set-up and the per-row index
// arithmetic are paid once for U chunks.  hidden is a multiple of E (the
// host checks a multiple of 4 and picks E = 8 for bf16 only when it is a
// multiple of 8), so every chunk is whole.
template <typename T, int E, int M, int U, int MAXIMG>
__device__ __forceinline__ void interp_block(const VisDesc<MAXIMG> &d, const InterpArgs &ia, int strip,
                                             int group, unsigned char *smem)
{
    constexpr int CS = interp_slice<T>();             // E: channels per lane access (4, or 8 for bf16)
    constexpr int NVM = CS / E;                       // lanes of one row slice (a power of two)
    constexpr int NV4 = CS / 4;                       // float4 of one slice of an R entry
    constexpr int NVU = U * NV4;                      // float4 of one R entry
    // image fields in registers (a dynamic index into the parameter block
    // would otherwise be re-read inside the loops)
    const int ii = find_image_of_strip(d, strip);
    const int im_t = d.img[ii].t, im_h = d.img[ii].h, im_w = d.img[ii].w, strip0 = d.img[ii].strip0;
    const long long row0 = d.img[ii].row0;
    const int m = M ? M : d.merge, G = d.grid_side, C = ia.hidden;
    float4 *R = reinterpret_cast<float4 *>(smem);
    int2 *cols = reinterpret_cast<int2 *>(smem + (size_t)m * G * NVU * sizeof(float4));
    int2 *rows = cols + kColCache;                    // the strip's m row samples
    const int by = strip - strip0;
    const int c0 = group * U * CS;
    const int nchunk = (min(U * CS, C - c0)) / E;     // chunks of this block (whole, see above)
    // Columns 0 .. x1 of the last sample: its point is G - 1 exactly when
    // w > 1 (x1 clipped to G - 1), and 0 when w = 1 (x1 = min(1, G - 1)).
    const int ncols = im_w > 1 ? G : min(2, G);
    const int v = threadIdx.x % NVM;
    const int rstep = blockDim.x / NVM;
    bool use[U];
#pragma unroll
    for (int u = 0; u < U; ++u) use[u] = u * NVM + v < nchunk;

    // Sample points once per block, packed as (i0 | i1 << 16, d): the
    // columns (phase 2 reads them back) and the strip's m rows.
    const bool cached = im_w <= kColCache;
    if (cached)
        for (int x = threadIdx.x; x < im_w; x += blockDim.x) {
            int x0, x1;
            float dx;
            grid_sample(x, im_w, G, x0, x1, dx);
            cols[x] = make_int2(x0 | (x1 << 16), __float_as_int(dx));
        }
    for (int iy = threadIdx.x; iy < m; iy += blockDim.x) {
        int y0, y1;
        float dy;
        grid_sample(by * m + iy, im_h, G, y0, y1, dy);
        rows[iy] = make_int2(y0 | (y1 << 16), __float_as_int(dy));
    }
    __syncthreads();

    // phase 1: y-blend of the strip's m patch rows.  R entry (iy, gx) holds
    // U x NV4 float4; lane v keeps chunk u at float4 u NV4 + v + NVM q, so
    // neighbouring lanes touch neighbouring banks in both phases.
    const T *tab_v = static_cast<const T *>(ia.table) + c0 + E * v;
    const int nrows = m * ncols;
    if (use[0]) {
        int r = threadIdx.x / NVM;
        int iy = r / ncols, gx = r - iy * ncols;
        for (; r < nrows; r += rstep) {
            const int2 rs = rows[iy];
            const int y0 = rs.x & 0xffff, y1 = rs.x >> 16;
            const float dy = __int_as_float(rs.y);
            const float2 DY = make_float2(dy, dy);
            const float omdy = __fsub_rn(1.f, dy);
            const float2 OMDY = make_float2(omdy, omdy);
            const T *ra = tab_v + (size_t)(y0 * G + gx) * C;
            const T *rb = tab_v + (size_t)(y1 * G + gx) * C;
            float4 *dst = R + r * NVU + v;
            float2 a[U][E / 2], b[U][E / 2];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (use[u]) {
                    load_pairs<T, E>(ra + u * CS, a[u]);
                    load_pairs<T, E>(rb + u * CS, b[u]);
                }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (use[u]) {
#pragma unroll
                    for (int q = 0; q < E / 4; ++q) {
                        // (1-dy) a + dy b, as fma(dy, b, (1-dy) a)
                        const float2 lo = fma2(DY, b[u][2 * q], mul2(OMDY, a[u][2 * q]));
                        const float2 hi = fma2(DY, b[u][2 * q + 1], mul2(OMDY, a[u][2 * q + 1]));
                        dst[u * NV4 + NVM * q] = make_float4(lo.x, lo.y, hi.x, hi.y);
                    }
                }
            gx += rstep;                           // next row of this thread
            while (gx >= ncols) {
                gx -= ncols;
                ++iy;
            }
        }
    }
    __syncthreads();

    // phase 2: x-blend, one rounding, every frame
    const size_t frame = (size_t)im_h * im_w * C;    // elements between frames
    T *out_v = static_cast<T *>(ia.out) + (size_t)(row0 + (long long)by * m * im_w) * C + c0 + E * v;
    if (use[0]) {
        for (int p = threadIdx.x / NVM; p < m * im_w; p += rstep) {
            int bx, iy, ix;                       // patch of the strip, merge order
            if constexpr (M == 2) {
                bx = p >> 2;
                iy = (p >> 1) & 1;
                ix = p & 1;
            } else {
                bx = p / (m * m);
                const int rr = p - bx * m * m;
                iy = rr / m;
                ix = rr - iy * m;
            }
            const int col = bx * m + ix;
            int x0, x1;
            float dx;
            if (cached) {
                const int2 cc = cols[col];
                x0 = cc.x & 0xffff;
                x1 = cc.x >> 16;
                dx = __int_as_float(cc.y);
            } else {
                grid_sample(col, im_w, G, x0, x1, dx);
            }
            const float2 DX = make_float2(dx, dx);
            const float omdx = __fsub_rn(1.f, dx);
            const float2 OMDX = make_float2(omdx, omdx);
            const float4 *r0 = R + (iy * ncols + x0) * NVU + v;
            const float4 *r1 = R + (iy * ncols + x1) * NVU + v;
            T *dst = out_v + (size_t)p * C;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (use[u]) {
                    float2 o[E / 2];
#pragma unroll
                    for (int q = 0; q < E / 4; ++q) {
                        const float4 a = r0[u * NV4 + NVM * q], b = r1[u * NV4 + NVM * q];
                        o[2 * q] = fma2(DX, make_float2(b.x, b.y), mul2(OMDX, make_float2(a.x, a.y)));
                        o[2 * q + 1] = fma2(DX, make_float2(b.z, b.w), mul2(OMDX, make_float2(a.z, a.w)));
                    }
#pragma unroll 1
                    for (int f = 0; f < im_t; ++f) store_pairs<T, E>(dst + u * CS + f * frame, o);
                }
        }
    }
}

// Resident blocks per SM the kernel is compiled for (merge 2, G = 48, bf16:
// the shared memory of U slices allows six blocks at U = 1, four at U = 2).
template <int U> constexpr int interp_min_blocks() { return U == 1 ? 6 : 4; }

template <typename T, int E, int M, int U, int MAXIMG>
__global__ void __launch_bounds__(kInterpThreads, interp_min_blocks<U>())
    vis_interp_kernel(const __grid_constant__ VisDesc<MAXIMG> d, const __grid_constant__ InterpArgs ia)
{
    extern __shared__ __align__(16) unsigned char smem[];
    interp_block<T, E, M, U, MAXIMG>(d, ia, blockIdx.x, blockIdx.y, smem);
}

// 16-byte accesses need 16-byte-aligned rows and base pointers.
template <typename T>
static bool interp_wide(const InterpArgs &ia)
{
    constexpr int E = 16 / (int)sizeof(T);
    return ia.hidden % E == 0 && (uintptr_t)ia.table % 16 == 0 && (uintptr_t)ia.out % 16 == 0;
}

// ------------------------------------------------------------- launches

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

// Slices per interpolation block: two when that grid still fills every SM
// twice at the occupancy its shared memory allows, else one.  Two slices
// share the block set-up and the row arithmetic (about a third fewer
// instructions on a batch of single images) but halve the blocks, which
// leaves SMs idle on small grids (a video's few strips, whose frames already
// amortise that work).  Measured on B200: a batch of 8 single images runs
// 28.4 us at one slice and 27.9 us at two; the 16 x 64 x 64 video, 42.0 and
// 42.8 us; three slices (two blocks per SM) were slower on both.
static int interp_pick_slices(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia)
{
    if (ia.n_slices < 2) return 1;
    const size_t smem = interp_smem_bytes(bf16, d.merge, d.grid_side, 2);
    if (smem > 227 * 1024) return 1;
    const long long per_sm = std::min<long long>(interp_min_blocks<2>(), 233472 / (long long)(smem + 1024));
    const long long blocks = (long long)d.n_strips * ((ia.n_slices + 1) / 2);
    return per_sm >= 1 && blocks >= 2 * per_sm * sm_count() ? 2 : 1;
}

template <typename T, int E, int M, int U, int MAXIMG>
static cudaError_t interp_launch(const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    const size_t smem = interp_smem_bytes(sizeof(T) == 2, d.merge, d.grid_side, U);
    auto kern = vis_interp_kernel<T, E, M, U, MAXIMG>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((unsigned)d.n_strips, (unsigned)((ia.n_slices + U - 1) / U));   // y <= n_slices <= 65535
    kern<<<grid, kInterpThreads, smem, s>>>(shrink<MAXIMG>(d), ia);
    return cudaGetLastError();
}

template <typename T, int E, int M, int MAXIMG>
static cudaError_t interp_slices(int u, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    if (u == 2) return interp_launch<T, E, M, 2, MAXIMG>(d, ia, s);
    return interp_launch<T, E, M, 1, MAXIMG>(d, ia, s);
}

template <typename T, int MAXIMG>
static cudaError_t interp_impl(const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    constexpr int EW = 16 / sizeof(T);
    const int u = interp_pick_slices(sizeof(T) == 2, d, ia);
    const bool wide = interp_wide<T>(ia), m2 = d.merge == 2;
    if (wide) return m2 ? interp_slices<T, EW, 2, MAXIMG>(u, d, ia, s) : interp_slices<T, EW, 0, MAXIMG>(u, d, ia, s);
    return m2 ? interp_slices<T, 4, 2, MAXIMG>(u, d, ia, s) : interp_slices<T, 4, 0, MAXIMG>(u, d, ia, s);
}

size_t vis_interp_block_smem(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia)
{
    return interp_smem_bytes(bf16, d.merge, d.grid_side, interp_pick_slices(bf16, d, ia));
}

cudaError_t launch_vis_interp(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    if (bf16)
        return d.n_images <= 16 ? interp_impl<__nv_bfloat16, 16>(d, ia, s) : interp_impl<__nv_bfloat16, 1024>(d, ia, s);
    return d.n_images <= 16 ? interp_impl<float, 16>(d, ia, s) : interp_impl<float, 1024>(d, ia, s);
}

template <typename T, int MAXIMG>
static cudaError_t rope_impl(const VisDesc<1024> &d, const RotArgs &r, const VisAngleFreqs &f, cudaStream_t s,
                             size_t budget)
{
    TmaRotArgs t;
    if (tma_rot_args(r, sizeof(T), t)) {
        t.aux_tma = 0;
        VisTmaSrc<MAXIMG> src{shrink<MAXIMG>(d), f};
        const int v = pick_vec(r, sizeof(T));
        if constexpr (sizeof(T) == 2) {
            if (v == 8) return launch_rotary_tma_vec<T, 8>(t, src, s, budget);
        }
        if (v >= 4) return launch_rotary_tma_vec<T, 4>(t, src, s, budget);
        return launch_rotary_tma_vec<T, 2>(t, src, s, budget);   // VEC >= 2 on the TMA path
    }
    VisSrc<MAXIMG> src{shrink<MAXIMG>(d), f};
    return dispatch_vec<T>(r, src, s);
}

cudaError_t launch_vis_rope(bool bf16, const VisDesc<1024> &d, const RotArgs &r, const VisAngleFreqs &f,
                            cudaStream_t s, size_t budget)
{
    if (budget == 0) budget = kTmaBlockSmem;
    if (bf16)
        return d.n_images <= 16 ? rope_impl<__nv_bfloat16, 16>(d, r, f, s, budget) : rope_impl<__nv_bfloat16, 1024>(d, r, f, s, budget);
    return d.n_images <= 16 ? rope_impl<float, 16>(d, r, f, s, budget) : rope_impl<float, 1024>(d, r, f, s, budget);
}

}  // namespace ipe
