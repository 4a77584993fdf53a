// Position-table interpolation in HF rounding mode: the rounding points of
// the "Qwen3-VL" notes' fast_pos_embed_interpolate listing, run as written in
// the table's dtype, for users who must match those checkpoints bit for bit.
//
//   * sample points: torch.linspace(0, G-1, n) in fp32.  Measured against
//     torch on the CPU (every n from 2 to 1024 at G = 48): the step
//     fl32((G-1)/(n-1)) once, then i * step for the first n/2 points and
//     (G-1) - (n-1-i) * step for the rest, each rounded once;
//   * corners by truncation and min(floor + 1, G - 1); dh = y - floor (fp32);
//   * weights (1-dh)(1-dw), (1-dh)dw, dh(1-dw), dh dw as fp32 products,
//     then stored in the table dtype;
//   * each corner row times its weight rounded to the dtype, and the four
//     products summed left to right, each sum taken in fp32 and rounded to
//     the dtype (how the dtype's elementwise arithmetic evaluates);
//   * frames repeat frame 0; rows in merge order.
//
// The default kernel (vis_interp_kernel) evaluates the separable form in
// fp32 with one rounding; this one evaluates the four-corner sum directly.
// A block takes a range of the patches of one merge-row strip of an image
// and 32 chunks of 16 bytes of the channels:
//   * set-up: each patch of its range gets its four corner rows and four
//     weights (rounded to the dtype) once, in shared memory;
//   * each warp then takes two output rows at a time (eight 16-byte table
//     loads in flight per lane), forms the four products and the
//     left-to-right sums, and writes each result chunk to every frame of
//     the video (frames repeat frame 0).
// The patch ranges split a strip over more blocks, so that a request of few
// strips still puts about eight blocks on every SM, while every block still
// reads each table value once for all of a video's frames.  For bf16 the products
// and sums run as packed bf16x2 operations, which round exactly where the
// fp32-then-round steps above do (mul_bf16x2 / add_bf16x2).
#include "ipe_internal.h"
#include "ipe_device.cuh"
#include "ipe_rotary.cuh"

namespace ipe {

constexpr int kHfWarps = 8;
constexpr int kHfPlanCache = 1024;   // strips of at most this many patches keep their plan in shared memory

// torch.linspace(0, G - 1, n)[i] in fp32.
__device__ __forceinline__ float hf_linspace(int i, int n, int G)
{
    if (n == 1) return 0.f;
    const float end = (float)(G - 1);
    const float step = __fdiv_rn(end, (float)(n - 1));
    if (i < n / 2) return __fmul_rn((float)i, step);
    return __fmaf_rn(-(float)(n - 1 - i), step, end);
}

// Corner table rows and weights of one output patch.  For bf16 the weights
// are bf16x2 words (the weight in both halves); for fp32 their bits.
struct HfPatch {
    int4 idx;
    uint4 w;
};

template <typename T>
__device__ __forceinline__ HfPatch hf_patch(int q, int sl, int m, int h, int w, int G)
{
    // merge order inside the strip: block column, then the m x m block row-major
    const int bx = q / (m * m), rr = q - bx * m * m;
    const int ih = sl * m + rr / m, iw = bx * m + rr % m;
    const float fy = hf_linspace(ih, h, G), fx = hf_linspace(iw, w, G);
    const int y0 = (int)fy, x0 = (int)fx;
    const int y1 = min(y0 + 1, G - 1), x1 = min(x0 + 1, G - 1);
    const float dh = __fsub_rn(fy, (float)y0), dw = __fsub_rn(fx, (float)x0);
    const float oh = __fsub_rn(1.f, dh), ow = __fsub_rn(1.f, dw);
    const float wt[4] = {round_to_dtype<T>(__fmul_rn(oh, ow)), round_to_dtype<T>(__fmul_rn(oh, dw)),
                         round_to_dtype<T>(__fmul_rn(dh, ow)), round_to_dtype<T>(__fmul_rn(dh, dw))};
    HfPatch p;
    p.idx = make_int4(y0 * G + x0, y0 * G + x1, y1 * G + x0, y1 * G + x1);
    uint32_t wb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if constexpr (sizeof(T) == 2) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(wt[k], wt[k]);   // exact: wt[k] is a bf16 value
            wb[k] = *reinterpret_cast<const uint32_t *>(&b);
        } else {
            wb[k] = __float_as_uint(wt[k]);
        }
    }
    p.w = make_uint4(wb[0], wb[1], wb[2], wb[3]);
    return p;
}

// One 16-byte chunk of an output row: the four products and the sums.
template <typename T>
__device__ __forceinline__ uint4 hf_blend(const uint4 (&c)[4], const uint4 &w)
{
    const uint32_t wk[4] = {w.x, w.y, w.z, w.w};
    if constexpr (sizeof(T) == 2) {
        const uint32_t cv[4][4] = {{c[0].x, c[0].y, c[0].z, c[0].w}, {c[1].x, c[1].y, c[1].z, c[1].w},
                                   {c[2].x, c[2].y, c[2].z, c[2].w}, {c[3].x, c[3].y, c[3].z, c[3].w}};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t acc = mul_bf16x2(cv[0][i], wk[0]);
#pragma unroll
            for (int k = 1; k < 4; ++k) acc = add_bf16x2(acc, mul_bf16x2(cv[k][i], wk[k]));
            o[i] = acc;
        }
        return make_uint4(o[0], o[1], o[2], o[3]);
    } else {
        const float cv[4][4] = {{__uint_as_float(c[0].x), __uint_as_float(c[0].y), __uint_as_float(c[0].z), __uint_as_float(c[0].w)},
                                {__uint_as_float(c[1].x), __uint_as_float(c[1].y), __uint_as_float(c[1].z), __uint_as_float(c[1].w)},
                                {__uint_as_float(c[2].x), __uint_as_float(c[2].y), __uint_as_float(c[2].z), __uint_as_float(c[2].w)},
                                {__uint_as_float(c[3].x), __uint_as_float(c[3].y), __uint_as_float(c[3].z), __uint_as_float(c[3].w)}};
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float acc = __fmul_rn(cv[0][e], __uint_as_float(wk[0]));
#pragma unroll
            for (int k = 1; k < 4; ++k) acc = __fadd_rn(acc, __fmul_rn(cv[k][e], __uint_as_float(wk[k])));
            o[e] = acc;
        }
        return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]), __float_as_uint(o[3]));
    }
}

template <typename T, int MAXIMG>
__global__ void __launch_bounds__(32 * kHfWarps) vis_interp_hf_kernel(const __grid_constant__ VisDesc<MAXIMG> d,
                                                                      const __grid_constant__ InterpArgs ia, int parts)
{
    __shared__ HfPatch plan[kHfPlanCache];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x;
    const VisImage im = d.img[find_image_of_strip(d, s)];
    const int m = d.merge, G = d.grid_side, h = im.h, w = im.w;
    const int sl = s - im.strip0;                     // merge-row strip within the frame
    const int nq = m * w;                             // patches of the strip
    const int per = (nq + parts - 1) / parts;         // this block's patches: [qa, qb)
    const int qa = blockIdx.z * per, qb = min(nq, qa + per);
    if (qa >= qb) return;                             // a narrow strip has fewer parts (whole block: no barrier yet)
    const bool cached = qb - qa <= kHfPlanCache;
    if (cached)
        for (int q = qa + threadIdx.x; q < qb; q += blockDim.x) plan[q - qa] = hf_patch<T>(q, sl, m, h, w, G);
    __syncthreads();
    constexpr int EC = 16 / sizeof(T);
    const int chunks = ia.hidden / EC;
    const int ch = blockIdx.y * 32 + lane;            // this lane's 16-byte chunk
    if (ch >= chunks) return;
    const long long hw = (long long)h * w;
    const uint4 *tab = reinterpret_cast<const uint4 *>(ia.table) + ch;
    uint4 *out = reinterpret_cast<uint4 *>(ia.out) + ch;
    const long long rstride = chunks;                 // uint4 per table / output row
    const long long row0 = im.row0 + (long long)sl * nq;
    for (int q = qa + warp; q < qb; q += 2 * kHfWarps) {
        const int q2 = q + kHfWarps;
        const bool two = q2 < qb;
        const HfPatch pa = cached ? plan[q - qa] : hf_patch<T>(q, sl, m, h, w, G);
        const HfPatch pb = two ? (cached ? plan[q2 - qa] : hf_patch<T>(q2, sl, m, h, w, G)) : pa;
        uint4 ca[4], cb[4];
        const int ia4[4] = {pa.idx.x, pa.idx.y, pa.idx.z, pa.idx.w};
        const int ib4[4] = {pb.idx.x, pb.idx.y, pb.idx.z, pb.idx.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) ca[k] = tab[ia4[k] * rstride];
#pragma unroll
        for (int k = 0; k < 4; ++k) cb[k] = tab[ib4[k] * rstride];
        const uint4 oa = hf_blend<T>(ca, pa.w), ob = hf_blend<T>(cb, pb.w);
#pragma unroll 1
        for (int f = 0; f < im.t; ++f) {
            out[(row0 + q + f * hw) * rstride] = oa;
            if (two) out[(row0 + q2 + f * hw) * rstride] = ob;
        }
    }
}

// Parts per strip: enough blocks for about eight per SM.  Four left the
// last partial wave a fifth of the time on the 16 x 64 x 64 video (640
// blocks on 148 SMs: 33.3 us against 31.9 us at eight; 30.7 against 28.8 us
// on a batch of 8 single images).
static int hf_parts(const VisDesc<1024> &d, long long blocks_xy)
{
    int max_nq = 1;
    for (int i = 0; i < d.n_images; ++i) max_nq = std::max(max_nq, d.merge * d.img[i].w);
    const long long want = 8LL * sm_count();
    long long parts = (want + blocks_xy - 1) / std::max<long long>(blocks_xy, 1);
    parts = std::max<long long>(1, std::min<long long>(parts, std::min(max_nq, 65535)));
    return (int)parts;
}

cudaError_t launch_vis_interp_hf(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    const int ec = bf16 ? 8 : 4;
    const unsigned gy = (unsigned)((ia.hidden / ec + 31) / 32);
    const int parts = hf_parts(d, (long long)d.n_strips * gy);
    const dim3 grid((unsigned)d.n_strips, gy, (unsigned)parts);
    const bool small = d.n_images <= 16;
    if (bf16) {
        if (small)
            vis_interp_hf_kernel<__nv_bfloat16, 16><<<grid, 32 * kHfWarps, 0, s>>>(shrink<16>(d), ia, parts);
        else
            vis_interp_hf_kernel<__nv_bfloat16, 1024><<<grid, 32 * kHfWarps, 0, s>>>(d, ia, parts);
    } else {
        if (small)
            vis_interp_hf_kernel<float, 16><<<grid, 32 * kHfWarps, 0, s>>>(shrink<16>(d), ia, parts);
        else
            vis_interp_hf_kernel<float, 1024><<<grid, 32 * kHfWarps, 0, s>>>(d, ia, parts);
    }
    return cudaGetLastError();
}

}  // namespace ipe
