// Fused QK-RMSNorm + multimodal RoPE, in place on Q and K.
//
// "M01 RMSNorm and multimodal RoPE (interleaved / chunked)" (kuanzhou.online),
// problem summary and hints: every head row is RMS-normalised in fp32, cast
// back to the activation dtype, multiplied by the norm weight (in that
// order), and then rotated like ipe_mrope_apply.  The note on vllm-omni there
// explains why the two are worth fusing: they run back to back on every
// q and k of every full-attention layer.
//
// One warp per token.  The warp writes the token's (cos, sin) pairs into its
// shared-memory slot once; each head row is then held by LPR = D / EC lanes
// (EC elements = 16 bytes per lane), its sum of squares reduced with
// shuffles inside those lanes, and the rotary partner of a chunk fetched from
// the lane half a rotary slice away.  All D channels are written back.
#include "ipe_rotary.cuh"

namespace ipe {

constexpr int kQkWarps = 8;
constexpr int kQkUnroll = 2;          // head rows per lane in flight

template <typename T> struct QkElem;
template <> struct QkElem<__nv_bfloat16> {
    static constexpr int EC = 8;
};
template <> struct QkElem<float> {
    static constexpr int EC = 4;
};

// Round to the activation dtype (identity for fp32).
__device__ __forceinline__ float round_dtype(float v, __nv_bfloat16 *) { return __bfloat162float(__float2bfloat16_rn(v)); }
__device__ __forceinline__ float round_dtype(float v, float *) { return v; }

template <typename T, int LPR>
__global__ void __launch_bounds__(32 * kQkWarps) qk_norm_mrope_kernel(const __grid_constant__ QkNormArgs n,
                                                                      const __grid_constant__ MropeAngles a)
{
    constexpr int EC = QkElem<T>::EC;
    constexpr int RPW = 32 / LPR;                     // head rows per warp access
    extern __shared__ float4 qk_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = n.half, rot = 2 * half, D = n.head_dim;
    float *cs_c = reinterpret_cast<float *>(qk_smem) + (size_t)warp * 2 * n.half_pad;
    float *cs_s = cs_c + n.half_pad;
    const int c = lane % LPR;                         // this lane's chunk of a row
    const int sub = lane / LPR;                       // which of the RPW rows
    const int e0 = c * EC;                            // first element of the chunk
    const bool rotary = e0 < rot;
    const bool first_half = e0 < half;
    const int j0 = first_half ? e0 : e0 - half;       // frequency of element e0
    const int partner = first_half ? lane + half / EC : lane - half / EC;

    // norm weights of this chunk, as fp32
    float wq[EC], wk[EC];
    {
        const Pack<T, EC> pq = ld_pack<T, EC>(static_cast<const T *>(n.q_weight) + e0);
        const Pack<T, EC> pk = ld_pack<T, EC>(static_cast<const T *>(n.k_weight) + e0);
#pragma unroll
        for (int e = 0; e < EC; ++e) {
            wq[e] = to_f32(pq.v[e]);
            wk[e] = to_f32(pk.v[e]);
        }
    }
    const int H = n.hq + n.hk;
    const long long stride = (long long)gridDim.x * kQkWarps;
    for (long long t = (long long)blockIdx.x * kQkWarps + warp; t < n.T; t += stride) {
        // (cos, sin) of every frequency of token t
        for (int j = lane; j < half; j += 32) {
            const int ax = mrope_axis(j, a.section, a.interleaved);
            const int pos = __ldg(a.positions + (long long)ax * a.T + t);
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            sincosf(angle, &cs_s[j], &cs_c[j]);
        }
        __syncwarp();
        float co[EC], si[EC];
        if (rotary) {
#pragma unroll
            for (int e = 0; e < EC; ++e) {
                co[e] = cs_c[j0 + e];
                si[e] = cs_s[j0 + e];
            }
        }
        for (int h0 = 0; h0 < H; h0 += RPW * kQkUnroll) {
            Pack<T, EC> x[kQkUnroll];
            T *ptr[kQkUnroll];
#pragma unroll
            for (int u = 0; u < kQkUnroll; ++u) {
                const int h = h0 + u * RPW + sub;
                ptr[u] = nullptr;
                if (h < H) {
                    ptr[u] = (h < n.hq ? static_cast<T *>(n.q) + t * n.q_stride + (long long)h * D
                                       : static_cast<T *>(n.k) + t * n.k_stride + (long long)(h - n.hq) * D) + e0;
                    x[u] = ld_pack<T, EC>(ptr[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kQkUnroll; ++u) {
                const int h = h0 + u * RPW + sub;
                // rows of one warp access are uniform in (h < H) per RPW group;
                // the shuffles below stay inside each row's LPR lanes
                float xf[EC];
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < EC; ++e) {
                    xf[e] = h < H ? to_f32(x[u].v[e]) : 0.f;
                    ss = __fmaf_rn(xf[e], xf[e], ss);
                }
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, LPR);
                const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)D), n.eps));
                const bool is_q = h < n.hq;
                float y[EC];
#pragma unroll
                for (int e = 0; e < EC; ++e) {
                    // cast back to the dtype first, then the weight (one more rounding)
                    const float xn = round_dtype(__fmul_rn(xf[e], r), (T *)nullptr);
                    y[e] = round_dtype(__fmul_rn(xn, is_q ? wq[e] : wk[e]), (T *)nullptr);
                }
                float yp[EC];
#pragma unroll
                for (int e = 0; e < EC; ++e) yp[e] = __shfl_sync(0xffffffffu, y[e], rotary ? partner : lane);
                Pack<T, EC> o;
#pragma unroll
                for (int e = 0; e < EC; ++e) {
                    float v = y[e];
                    if (rotary)   // x[j] cos - x[j+h] sin ; x[j+h] cos + x[j] sin
                        v = first_half ? __fmaf_rn(y[e], co[e], -__fmul_rn(yp[e], si[e]))
                                       : __fmaf_rn(y[e], co[e], __fmul_rn(yp[e], si[e]));
                    o.v[e] = from_f32<T>(v);
                }
                if (ptr[u]) st_pack<T, EC>(ptr[u], o);
            }
        }
        __syncwarp();
    }
}

template <typename T, int LPR>
static cudaError_t qk_launch(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    const size_t smem = (size_t)kQkWarps * 2 * n.half_pad * sizeof(float);
    auto kern = qk_norm_mrope_kernel<T, LPR>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kQkWarps, smem);
    if (e != cudaSuccess) return e;
    const long long need = (n.T + kQkWarps - 1) / kQkWarps;
    const int blocks = (int)std::max<long long>(1, std::min(need, (long long)sm_count() * std::max(per_sm, 1)));
    kern<<<blocks, 32 * kQkWarps, smem, s>>>(n, a);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t qk_dispatch(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    switch (n.head_dim / QkElem<T>::EC) {
    case 32: return qk_launch<T, 32>(n, a, s);
    case 16: return qk_launch<T, 16>(n, a, s);
    case 8: return qk_launch<T, 8>(n, a, s);
    case 4: return qk_launch<T, 4>(n, a, s);
    case 2: return qk_launch<T, 2>(n, a, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_qk_norm_mrope(bool bf16, const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    return bf16 ? qk_dispatch<__nv_bfloat16>(n, a, s) : qk_dispatch<float>(n, a, s);
}

}  // namespace ipe
