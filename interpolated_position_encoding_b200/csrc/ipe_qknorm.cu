// Fused QK-RMSNorm + multimodal RoPE, in place on Q and K.
//
// "M01 RMSNorm and multimodal RoPE (interleaved / chunked)" (kuanzhou.online),
// problem summary and hints: every head row is RMS-normalised in fp32, cast
// back to the activation dtype, multiplied by the norm weight (in that
// order), and then rotated like ipe_mrope_apply.  The note on vllm-omni there
// explains why the two are worth fusing: they run back to back on every
// q and k of every full-attention layer.
//
// One warp per token (for short sequences, per token and group of head rows).
// The warp writes the token's (cos, sin) pairs into its shared-memory slot once; each head row is then held by LPR = D / EC lanes
// (EC elements = 16 bytes per lane), its sum of squares reduced with
// shuffles inside those lanes, and the rotary partner of a chunk fetched from
// the lane half a rotary slice away.  All D channels are written back.
#include "ipe_chunk.cuh"

namespace ipe {

constexpr int kQkWarps = 8;
// Rows in flight per lane and blocks per SM, by lanes per row (measured:
// 256-channel bf16 rows prefer four rows at three blocks per SM, narrower
// rows two rows at four blocks per SM).
constexpr int qk_unroll(int lpr) { return lpr >= 32 ? 4 : 2; }
constexpr int qk_min_blocks(int lpr) { return lpr >= 32 ? 3 : 4; }

template <typename T, int LPR>
__global__ void __launch_bounds__(32 * kQkWarps, qk_min_blocks(LPR))
    qk_norm_mrope_kernel(const __grid_constant__ QkNormArgs n, const __grid_constant__ MropeAngles a)
{
    constexpr int EC = QkElem<T>::EC;
    constexpr int NP = EC / 2;                        // fp32 pairs of a 16-byte chunk
    constexpr int kQkUnroll = qk_unroll(LPR);
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
    const int partner = rotary ? (first_half ? lane + half / EC : lane - half / EC) : lane;
    // D = LPR * EC is a power of two: multiplying by 1/D is the exact division
    const float inv_d = __frcp_rn((float)D);

    // norm weights of this chunk, as words
    const Pack<uint32_t, 4> wq = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(static_cast<const T *>(n.q_weight) + e0));
    const Pack<uint32_t, 4> wk = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(static_cast<const T *>(n.k_weight) + e0));
    const int H = n.hq + n.hk;
    // this warp's group of head rows (the grid holds a multiple of `groups`
    // warps, so the group stays fixed while the warp strides over tokens)
    const int gw = blockIdx.x * kQkWarps + warp;
    const int hbeg = (gw % n.groups) * n.rows_per_item;
    const int hend = min(H, hbeg + n.rows_per_item);
    const long long tstride = (long long)gridDim.x * kQkWarps / n.groups;
    for (long long t = gw / n.groups; t < n.T; t += tstride) {
        Pack<uint32_t, 4> x[kQkUnroll];
        // this lane's chunk of head row h of token t
        auto chunk_ptr = [&](int h) {
            T *row = h < n.hq ? static_cast<T *>(n.q) + t * n.q_stride + (long long)h * D
                              : static_cast<T *>(n.k) + t * n.k_stride + (long long)(h - n.hq) * D;
            return reinterpret_cast<uint32_t *>(row + e0);
        };
        // rows h0 + u * RPW + sub of token t (zeros past the item's last row)
        auto load_group = [&](int h0) {
#pragma unroll
            for (int u = 0; u < kQkUnroll; ++u) {
                const int h = h0 + u * RPW + sub;
                if (h < hend) {
                    x[u] = ld_pack<uint32_t, 4>(chunk_ptr(h));
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) x[u].v[i] = 0u;
                }
            }
        };
        // the first rows are in flight while the angles are computed
        load_group(hbeg);
        // (cos, sin) of every frequency of token t
        for (int j = lane; j < half; j += 32) {
            const int ax = mrope_axis(j, a.section, a.interleaved);
            const int pos = __ldg(a.positions + (long long)ax * a.T + t);
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            sincosf(angle, &cs_s[j], &cs_c[j]);
        }
        __syncwarp();
        // cos and the signed sine of this chunk (pass-through: 1 and 0)
        float2 co[NP], si[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            co[i] = rotary ? make_float2(cs_c[j0 + 2 * i], cs_c[j0 + 2 * i + 1]) : make_float2(1.f, 1.f);
            const float2 sv = rotary ? make_float2(cs_s[j0 + 2 * i], cs_s[j0 + 2 * i + 1]) : make_float2(0.f, 0.f);
            si[i] = first_half ? make_float2(-sv.x, -sv.y) : sv;
        }
        for (int h0 = hbeg; h0 < hend; h0 += RPW * kQkUnroll) {
            if (h0 > hbeg) load_group(h0);
#pragma unroll
            for (int u = 0; u < kQkUnroll; ++u) {
                // every lane of the warp takes part in the shuffles, rows past
                // the item's last included (zeros; never stored)
                const int h = h0 + u * RPW + sub;
                const bool is_q = h < n.hq;
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = is_q ? wq.v[i] : wk.v[i];
                const Pack<uint32_t, 4> y = rms_norm_chunk<T, LPR>(x[u], w, inv_d, n.eps);
                const Pack<uint32_t, 4> o = rotate_row_chunk<T>(y, co, si, partner);
                if (h < hend) st_pack<uint32_t, 4>(chunk_ptr(h), o);
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
    // Short sequences: a token's head rows are split over several warps
    // (whole passes of RPW x unroll rows each) until there are about four
    // warps per resident warp slot; long ones keep one warp per token.
    QkNormArgs m = n;
    const int unit = (32 / LPR) * qk_unroll(LPR);
    const int H = n.hq + n.hk;
    const int max_groups = (H + unit - 1) / unit;
    const long long want = 4LL * sm_count() * std::max(per_sm, 1) * kQkWarps;
    int groups = 1;
    while (groups < max_groups && n.T * groups < want) ++groups;
    m.rows_per_item = ((H + groups - 1) / groups + unit - 1) / unit * unit;
    m.groups = (H + m.rows_per_item - 1) / m.rows_per_item;
    const long long need = (n.T * m.groups + kQkWarps - 1) / kQkWarps;
    long long blocks = std::max<long long>(1, std::min(need, (long long)sm_count() * std::max(per_sm, 1)));
    blocks = (blocks + m.groups - 1) / m.groups * m.groups;   // a whole number of groups per stride
    kern<<<(unsigned)blocks, 32 * kQkWarps, smem, s>>>(m, a);
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
