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
// fp32 with one rounding; this one evaluates the four-corner sum directly:
// a block takes one merge-row strip of frame 0 and 32 chunks of 16 bytes of
// the channels, each warp one output row at a time, and each result chunk
// is written once per frame.  For bf16 the products and sums run as packed
// bf16x2 operations, which round exactly where the fp32-then-round steps
// above do (mul_bf16x2 / add_bf16x2).
#include "ipe_internal.h"
#include "ipe_device.cuh"

namespace ipe {

constexpr int kHfWarps = 8;

// torch.linspace(0, G - 1, n)[i] in fp32.
__device__ __forceinline__ float hf_linspace(int i, int n, int G)
{
    if (n == 1) return 0.f;
    const float end = (float)(G - 1);
    const float step = __fdiv_rn(end, (float)(n - 1));
    if (i < n / 2) return __fmul_rn((float)i, step);
    return __fmaf_rn(-(float)(n - 1 - i), step, end);
}

template <typename T>
__global__ void __launch_bounds__(32 * kHfWarps) vis_interp_hf_kernel(const __grid_constant__ VisDesc<1024> d,
                                                                      const __grid_constant__ InterpArgs ia)
{
    constexpr int EC = 16 / sizeof(T);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x;
    const VisImage im = d.img[find_image_of_strip(d, s)];
    const int m = d.merge, G = d.grid_side, h = im.h, w = im.w;
    const int sl = s - im.strip0;                     // merge-row strip within the frame
    const int chunks = ia.hidden / EC;
    const int ch = blockIdx.y * 32 + lane;            // this lane's 16-byte chunk
    const long long hw = (long long)h * w;
    const T *table = static_cast<const T *>(ia.table);
    T *out = static_cast<T *>(ia.out);
    for (int q = warp; q < m * w; q += kHfWarps) {
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
        const long long idx[4] = {(long long)y0 * G + x0, (long long)y0 * G + x1, (long long)y1 * G + x0,
                                  (long long)y1 * G + x1};
        if (ch >= chunks) continue;
        const long long row = im.row0 + (long long)sl * m * w + q;
        if constexpr (sizeof(T) == 2) {
            // eight bf16 channels as four bf16x2 words; weights broadcast to both halves
            Pack<uint32_t, 4> c[4], o;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                c[k] = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(table + idx[k] * ia.hidden) + ch * 4);
            uint32_t w2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(wt[k], wt[k]);   // exact: wt[k] is a bf16 value
                w2[k] = *reinterpret_cast<const uint32_t *>(&b);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t acc = mul_bf16x2(c[0].v[i], w2[0]);
#pragma unroll
                for (int k = 1; k < 4; ++k) acc = add_bf16x2(acc, mul_bf16x2(c[k].v[i], w2[k]));
                o.v[i] = acc;
            }
#pragma unroll 1
            for (int f = 0; f < im.t; ++f)
                st_pack<uint32_t, 4>(reinterpret_cast<uint32_t *>(out + (row + f * hw) * ia.hidden) + ch * 4, o);
        } else {
            Pack<T, EC> c[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) c[k] = ld_pack<T, EC>(table + idx[k] * ia.hidden + (long long)ch * EC);
            Pack<T, EC> o;
#pragma unroll
            for (int e = 0; e < EC; ++e) {
                float acc = round_to_dtype<T>(__fmul_rn(to_f32(c[0].v[e]), wt[0]));
#pragma unroll
                for (int k = 1; k < 4; ++k)
                    acc = round_to_dtype<T>(__fadd_rn(acc, round_to_dtype<T>(__fmul_rn(to_f32(c[k].v[e]), wt[k]))));
                o.v[e] = from_f32<T>(acc);
            }
#pragma unroll 1
            for (int f = 0; f < im.t; ++f) st_pack<T, EC>(out + (row + f * hw) * ia.hidden + (long long)ch * EC, o);
        }
    }
}

cudaError_t launch_vis_interp_hf(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s)
{
    const int ec = bf16 ? 8 : 4;
    const dim3 grid((unsigned)d.n_strips, (unsigned)((ia.hidden / ec + 31) / 32));
    if (bf16)
        vis_interp_hf_kernel<__nv_bfloat16><<<grid, 32 * kHfWarps, 0, s>>>(d, ia);
    else
        vis_interp_hf_kernel<float><<<grid, 32 * kHfWarps, 0, s>>>(d, ia);
    return cudaGetLastError();
}

}  // namespace ipe
