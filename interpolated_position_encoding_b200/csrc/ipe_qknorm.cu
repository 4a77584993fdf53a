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
// The warp writes the token's (cos, sin) pairs into its shared-memory slot
// once.  Three lane layouts of a head row (EC elements = 16 bytes per chunk):
//   * qk_norm_mrope_split_kernel, for a rotary slice narrower than the row:
//     rot / EC lanes, D / rot chunks each, so that only a lane's first chunk
//     is rotated;
//   * qk_norm_mrope_pair_kernel, for a rotary slice as wide as the row:
//     D / (2 EC) lanes, each with a chunk of either half, so that both
//     members of a rotation pair sit in one lane;
//   * qk_norm_mrope_kernel otherwise: LPR = D / EC lanes, one chunk each.
// The row's sum of squares is reduced with shuffles inside its lanes, and
// the rotary partner of a chunk is fetched from the lane half a rotary slice
// away.  All D channels are written back.
#include "ipe_chunk.cuh"

namespace ipe {

constexpr int kQkWarps = 8;
// Pair layout: row groups in flight per warp (U) and blocks per SM.
// Measured on B200 (Qwen3-Omni, T = 32768, 36 rows of 128 channels): one
// group at four blocks per SM 106.2 us, two at three 103.7 us, three at
// three 101.7 us, three at two 100.7 us; four or six (rows padded to 48)
// 113 us.
constexpr int qk_pair_min_blocks(int u) { return u >= 3 ? 2 : 3; }
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
    // x[u] holds row hbeg + u RPW + sub (+ a multiple of RPW x unroll) of the
    // token in hand; as soon as a slot's row is written back the slot loads
    // its row of the next group, or of this warp's next token, so the loads
    // stay in flight while the norms, rotations and stores run.
    Pack<uint32_t, 4> x[kQkUnroll];
    // this lane's chunk of head row h of token t
    auto chunk_ptr = [&](long long t, int h) {
        T *row = h < n.hq ? static_cast<T *>(n.q) + t * n.q_stride + (long long)h * D
                          : static_cast<T *>(n.k) + t * n.k_stride + (long long)(h - n.hq) * D;
        return reinterpret_cast<uint32_t *>(row + e0);
    };
    auto load_row = [&](long long t, int h, Pack<uint32_t, 4> &v) {
        if (t < n.T && h < hend) {
            v = ld_pack<uint32_t, 4>(chunk_ptr(t, h));
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) v.v[i] = 0u;   // past the item's last row: zeros, never stored
        }
    };
    long long t = gw / n.groups;
#pragma unroll
    for (int u = 0; u < kQkUnroll; ++u) load_row(t, hbeg + u * RPW + sub, x[u]);
    for (; t < n.T; t += tstride) {
        // (cos, sin) of every frequency of token t, while its rows load
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
            const bool last = h0 + RPW * kQkUnroll >= hend;
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
                if (h < hend) st_pack<uint32_t, 4>(chunk_ptr(t, h), o);
                if (last)
                    load_row(t + tstride, hbeg + u * RPW + sub, x[u]);
                else
                    load_row(t, h + RPW * kQkUnroll, x[u]);
            }
        }
        __syncwarp();
    }
}

// Rows whose rotary slice is narrower than the row (rot < D, rot / EC a
// power of two): LPR = rot / EC lanes per head row, each holding the CPL =
// D / rot chunks c, c + LPR, ... of it (a stride of rot channels).  A lane's
// first chunk lies in the rotary slice and the others pass through, so the
// rotation (partner shuffle and arithmetic) runs on one chunk in CPL instead
// of on every chunk, and the sum of squares is reduced over LPR lanes.  Each
// chunk's norm, cast and weight product are those of the kernel above; only
// the order in which the row's squares are summed differs.  The norm weights
// sit in shared memory; the next row of a lane's CPL chunks is loaded while
// the current one is worked on.  MINB blocks per SM: three keep more warps
// on short sequences, two leave bf16 rows of four chunks per lane their
// registers (at three they spill) for long ones.  Measured on B200, bf16
// D = 256, rot 64: 131072 tokens 606 us at three against 584 us at two;
// 4096 tokens 24.3 us against 33.5 us.
template <typename T, int LPR, int CPL, int MINB>
__global__ void __launch_bounds__(32 * kQkWarps, MINB)
    qk_norm_mrope_split_kernel(const __grid_constant__ QkNormArgs n, const __grid_constant__ MropeAngles a)
{
    constexpr int EC = QkElem<T>::EC;
    constexpr int NP = EC / 2;                        // fp32 pairs of a 16-byte chunk
    constexpr int RPW = 32 / LPR;                     // head rows per warp access
    constexpr int ROT = LPR * EC;                     // rotary channels
    constexpr int D = ROT * CPL;
    constexpr int WCH = D / EC;                       // chunks of one weight vector
    extern __shared__ float4 qk_smem[];
    uint4 *wsm = reinterpret_cast<uint4 *>(qk_smem);  // q weights, then k weights
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *cs_c = reinterpret_cast<float *>(wsm + 2 * WCH) + (size_t)warp * 2 * n.half_pad;
    float *cs_s = cs_c + n.half_pad;
    for (int i = threadIdx.x; i < 2 * WCH; i += blockDim.x)
        wsm[i] = *reinterpret_cast<const uint4 *>(i < WCH ? static_cast<const T *>(n.q_weight) + i * EC
                                                          : static_cast<const T *>(n.k_weight) + (i - WCH) * EC);
    __syncthreads();
    constexpr int half = ROT / 2;
    const int c = lane % LPR;                         // this lane's rotary chunk
    const int sub = lane / LPR;                       // which of the RPW rows
    const int e0 = c * EC;
    const bool first_half = e0 < half;
    const int j0 = first_half ? e0 : e0 - half;       // frequency of element e0
    const int partner = first_half ? lane + half / EC : lane - half / EC;
    const float inv_d = __frcp_rn((float)D);          // D a power of two: exact
    const int H = n.hq + n.hk;
    const int gw = blockIdx.x * kQkWarps + warp;
    const int hbeg = (gw % n.groups) * n.rows_per_item;
    const int hend = min(H, hbeg + n.rows_per_item);
    const long long tstride = (long long)gridDim.x * kQkWarps / n.groups;
    auto row_ptr = [&](long long t, int h) {
        T *row = h < n.hq ? static_cast<T *>(n.q) + t * n.q_stride + (long long)h * D
                          : static_cast<T *>(n.k) + t * n.k_stride + (long long)(h - n.hq) * D;
        return reinterpret_cast<uint32_t *>(row + e0);
    };
    // this lane's CPL chunks of row h of token t (zeros past the item's rows)
    auto load_row = [&](long long t, int h, Pack<uint32_t, 4> *v) {
        if (t < n.T && h < hend) {
            const uint32_t *p = row_ptr(t, h);
#pragma unroll
            for (int k = 0; k < CPL; ++k) v[k] = ld_pack<uint32_t, 4>(p + k * (ROT * (int)sizeof(T) / 4));
        } else {
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
                for (int i = 0; i < 4; ++i) v[k].v[i] = 0u;
        }
    };
    long long t = gw / n.groups;
    Pack<uint32_t, 4> x[CPL];
    load_row(t, hbeg + sub, x);
    for (; t < n.T; t += tstride) {
        // (cos, sin) of every frequency of token t
        for (int j = lane; j < half; j += 32) {
            const int ax = mrope_axis(j, a.section, a.interleaved);
            const int pos = __ldg(a.positions + (long long)ax * a.T + t);
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            sincosf(angle, &cs_s[j], &cs_c[j]);
        }
        __syncwarp();
        float2 co[NP], si[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            co[i] = make_float2(cs_c[j0 + 2 * i], cs_c[j0 + 2 * i + 1]);
            const float2 sv = make_float2(cs_s[j0 + 2 * i], cs_s[j0 + 2 * i + 1]);
            si[i] = first_half ? make_float2(-sv.x, -sv.y) : sv;
        }
        for (int h0 = hbeg; h0 < hend; h0 += RPW) {
            const int h = h0 + sub;
            // the next row (of this token, or of the next one) is loaded now
            Pack<uint32_t, 4> nx[CPL];
            if (h0 + RPW < hend)
                load_row(t, h + RPW, nx);
            else
                load_row(t + tstride, hbeg + sub, nx);
            // every lane of the warp takes part in the shuffles
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                float2 xv[NP];
                chunk_to_pairs<T>(x[k].v, xv);
#pragma unroll
                for (int i = 0; i < NP; ++i) acc = (k == 0 && i == 0) ? mul2(xv[0], xv[0]) : fma2(xv[i], xv[i], acc);
            }
            float ss = __fadd_rn(acc.x, acc.y);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, LPR);
            const float r = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, inv_d), n.eps));
            const float2 r2 = make_float2(r, r);
            const uint4 *wrow = wsm + (h < n.hq ? 0 : WCH) + c;
            Pack<uint32_t, 4> y[CPL];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                // cast back first, then the weight
                float2 xv[NP];
                chunk_to_pairs<T>(x[k].v, xv);
#pragma unroll
                for (int i = 0; i < NP; ++i) xv[i] = mul2(xv[i], r2);
                pairs_to_chunk<T>(xv, y[k].v);
                const uint4 wv = wrow[k * LPR];
                const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
                if constexpr (std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) y[k].v[i] = mul_bf16x2(y[k].v[i], w[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        y[k].v[i] = __float_as_uint(__fmul_rn(__uint_as_float(y[k].v[i]), __uint_as_float(w[i])));
                }
            }
            y[0] = rotate_row_chunk<T>(y[0], co, si, partner);
            if (h < hend) {
                uint32_t *p = row_ptr(t, h);
#pragma unroll
                for (int k = 0; k < CPL; ++k) st_pack<uint32_t, 4>(p + k * (ROT * (int)sizeof(T) / 4), y[k]);
            }
#pragma unroll
            for (int k = 0; k < CPL; ++k) x[k] = nx[k];
        }
        __syncwarp();
    }
}

// Warps over tokens and head-row groups (shared by both kernels): a token's
// head rows are split over several warps (whole passes of `unit` rows each)
// until there are about four warps per resident warp slot; long sequences
// keep one warp per token.
static void qk_grid(QkNormArgs &m, int unit, int per_sm, long long &blocks)
{
    const int H = m.hq + m.hk;
    const int max_groups = (H + unit - 1) / unit;
    const long long want = 4LL * sm_count() * std::max(per_sm, 1) * kQkWarps;
    int groups = 1;
    while (groups < max_groups && m.T * groups < want) ++groups;
    m.rows_per_item = ((H + groups - 1) / groups + unit - 1) / unit * unit;
    m.groups = (H + m.rows_per_item - 1) / m.rows_per_item;
    const long long need = (m.T * m.groups + kQkWarps - 1) / kQkWarps;
    blocks = std::max<long long>(1, std::min(need, (long long)sm_count() * std::max(per_sm, 1)));
    blocks = (blocks + m.groups - 1) / m.groups * m.groups;   // a whole number of groups per stride
}

// Rows whose rotary slice is the whole row (rot = D, Qwen3-Omni): LPR =
// half / EC lanes per head row, each holding chunk c of the first half and
// chunk c of the second half (elements e0 + j and e0 + half + j).  Both
// members of every rotation pair then sit in the same lane, so the rotation
// needs no partner shuffle, and the sum of squares is reduced over LPR
// lanes instead of D / EC.  The norm, cast, weight product and rotation are
// those of the kernels above; only the order in which the row's squares are
// summed differs.
template <typename T, int LPR, int U>
__global__ void __launch_bounds__(32 * kQkWarps, qk_pair_min_blocks(U))
    qk_norm_mrope_pair_kernel(const __grid_constant__ QkNormArgs n, const __grid_constant__ MropeAngles a)
{
    constexpr int EC = QkElem<T>::EC;
    constexpr int NP = EC / 2;                        // fp32 pairs of a 16-byte chunk
    constexpr int RPW = 32 / LPR;                     // head rows per warp access
    constexpr int HALF = LPR * EC;
    constexpr int D = 2 * HALF;
    constexpr int WCH = D / EC;                       // chunks of one weight vector
    extern __shared__ float4 qk_smem[];
    uint4 *wsm = reinterpret_cast<uint4 *>(qk_smem);  // q weights, then k weights
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *cs_c = reinterpret_cast<float *>(wsm + 2 * WCH) + (size_t)warp * 2 * n.half_pad;
    float *cs_s = cs_c + n.half_pad;
    for (int i = threadIdx.x; i < 2 * WCH; i += blockDim.x)
        wsm[i] = *reinterpret_cast<const uint4 *>(i < WCH ? static_cast<const T *>(n.q_weight) + i * EC
                                                          : static_cast<const T *>(n.k_weight) + (i - WCH) * EC);
    __syncthreads();
    const int c = lane % LPR;                         // this lane's chunk of each half
    const int sub = lane / LPR;                       // which of the RPW rows
    const int e0 = c * EC;
    const float inv_d = __frcp_rn((float)D);          // D a power of two: exact
    const int H = n.hq + n.hk;
    const int gw = blockIdx.x * kQkWarps + warp;
    const int hbeg = (gw % n.groups) * n.rows_per_item;
    const int hend = min(H, hbeg + n.rows_per_item);
    const long long tstride = (long long)gridDim.x * kQkWarps / n.groups;
    constexpr int kHalfWords = HALF * (int)sizeof(T) / 4;
    auto row_ptr = [&](long long t, int h) {
        T *row = h < n.hq ? static_cast<T *>(n.q) + t * n.q_stride + (long long)h * D
                          : static_cast<T *>(n.k) + t * n.k_stride + (long long)(h - n.hq) * D;
        return reinterpret_cast<uint32_t *>(row + e0);
    };
    auto load_row = [&](long long t, int h, Pack<uint32_t, 4> *v) {
        if (t < n.T && h < hend) {
            const uint32_t *p = row_ptr(t, h);
            v[0] = ld_pack<uint32_t, 4>(p);
            v[1] = ld_pack<uint32_t, 4>(p + kHalfWords);
        } else {
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int i = 0; i < 4; ++i) v[k].v[i] = 0u;
        }
    };
    // U slots of row groups: slot u holds row h0 + u RPW + sub of the token
    // in hand and, as soon as it is taken for the norm, loads the row it will
    // hold next (U RPW rows further, or the next token's), so U groups of
    // loads stay in flight per warp
    long long t = gw / n.groups;
    Pack<uint32_t, 4> x[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) load_row(t, hbeg + u * RPW + sub, x[u]);
    for (; t < n.T; t += tstride) {
        // (cos, sin) of every frequency of token t
        for (int j = lane; j < HALF; j += 32) {
            const int ax = mrope_axis(j, a.section, a.interleaved);
            const int pos = __ldg(a.positions + (long long)ax * a.T + t);
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            sincosf(angle, &cs_s[j], &cs_c[j]);
        }
        __syncwarp();
        float2 co[NP], sn[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            co[i] = make_float2(cs_c[e0 + 2 * i], cs_c[e0 + 2 * i + 1]);
            sn[i] = make_float2(cs_s[e0 + 2 * i], cs_s[e0 + 2 * i + 1]);
        }
        for (int h0 = hbeg; h0 < hend; h0 += RPW * U) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = h0 + u * RPW + sub;
                float2 xa[NP], xb[NP];
                chunk_to_pairs<T>(x[u][0].v, xa);
                chunk_to_pairs<T>(x[u][1].v, xb);
                if (h0 + RPW * U < hend)
                    load_row(t, h + RPW * U, x[u]);
                else
                    load_row(t + tstride, hbeg + u * RPW + sub, x[u]);
                float2 acc = mul2(xa[0], xa[0]);
#pragma unroll
                for (int i = 1; i < NP; ++i) acc = fma2(xa[i], xa[i], acc);
#pragma unroll
                for (int i = 0; i < NP; ++i) acc = fma2(xb[i], xb[i], acc);
                float ss = __fadd_rn(acc.x, acc.y);
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, LPR);
                const float r = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, inv_d), n.eps));
                const float2 r2 = make_float2(r, r);
                const uint4 *wrow = wsm + (h < n.hq ? 0 : WCH) + c;
                // cast back first, then the weight (both halves)
                Pack<uint32_t, 4> ya, yb;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    xa[i] = mul2(xa[i], r2);
                    xb[i] = mul2(xb[i], r2);
                }
                pairs_to_chunk<T>(xa, ya.v);
                pairs_to_chunk<T>(xb, yb.v);
                const uint4 wa = wrow[0], wb = wrow[LPR];
                const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w}, wbv[4] = {wb.x, wb.y, wb.z, wb.w};
                if constexpr (std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        ya.v[i] = mul_bf16x2(ya.v[i], wav[i]);
                        yb.v[i] = mul_bf16x2(yb.v[i], wbv[i]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        ya.v[i] = __float_as_uint(__fmul_rn(__uint_as_float(ya.v[i]), __uint_as_float(wav[i])));
                        yb.v[i] = __float_as_uint(__fmul_rn(__uint_as_float(yb.v[i]), __uint_as_float(wbv[i])));
                    }
                }
                // x'[j] = x[j] cos_j - x[j+h] sin_j,  x'[j+h] = x[j+h] cos_j + x[j] sin_j
                float2 va[NP], vb[NP], oa[NP], ob[NP];
                chunk_to_pairs<T>(ya.v, va);
                chunk_to_pairs<T>(yb.v, vb);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const float2 ns = make_float2(-sn[i].x, -sn[i].y);
                    oa[i] = fma2(va[i], co[i], mul2(vb[i], ns));
                    ob[i] = fma2(vb[i], co[i], mul2(va[i], sn[i]));
                }
                Pack<uint32_t, 4> pa, pb;
                pairs_to_chunk<T>(oa, pa.v);
                pairs_to_chunk<T>(ob, pb.v);
                if (h < hend) {
                    uint32_t *p = row_ptr(t, h);
                    st_pack<uint32_t, 4>(p, pa);
                    st_pack<uint32_t, 4>(p + kHalfWords, pb);
                }
            }
        }
        __syncwarp();
    }
}

template <typename T, int LPR, int U>
static cudaError_t qk_launch_pair_u(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    constexpr int EC = QkElem<T>::EC;
    const size_t smem = 2 * (size_t)2 * LPR * EC * sizeof(T) + (size_t)kQkWarps * 2 * n.half_pad * sizeof(float);
    auto kern = qk_norm_mrope_pair_kernel<T, LPR, U>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kQkWarps, smem);
    if (e != cudaSuccess) return e;
    QkNormArgs m = n;
    long long blocks = 0;
    qk_grid(m, (32 / LPR) * U, per_sm, blocks);
    kern<<<(unsigned)blocks, 32 * kQkWarps, smem, s>>>(m, a);
    return cudaGetLastError();
}

// Three groups in flight unless two pad the head rows less (the rows past
// the last are zeros that are never stored, but still cost their work).
template <typename T, int LPR>
static cudaError_t qk_launch_pair(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    constexpr int RPW = 32 / LPR;
    const int H = n.hq + n.hk;
    auto pad = [&](int u) { return (H + RPW * u - 1) / (RPW * u) * (RPW * u) - H; };
    return pad(2) < pad(3) ? qk_launch_pair_u<T, LPR, 2>(n, a, s) : qk_launch_pair_u<T, LPR, 3>(n, a, s);
}

template <typename T, int LPR, int CPL, int MINB>
static cudaError_t qk_launch_split(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    constexpr int EC = QkElem<T>::EC;
    const size_t smem = 2 * (size_t)LPR * CPL * EC * sizeof(T) + (size_t)kQkWarps * 2 * n.half_pad * sizeof(float);
    auto kern = qk_norm_mrope_split_kernel<T, LPR, CPL, MINB>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kQkWarps, smem);
    if (e != cudaSuccess) return e;
    QkNormArgs m = n;
    long long blocks = 0;
    qk_grid(m, 32 / LPR, per_sm, blocks);
    kern<<<(unsigned)blocks, 32 * kQkWarps, smem, s>>>(m, a);
    return cudaGetLastError();
}

template <typename T, int LPR>
static cudaError_t qk_launch(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    const size_t smem = (size_t)kQkWarps * 2 * n.half_pad * sizeof(float);
    auto kern = qk_norm_mrope_kernel<T, LPR>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kQkWarps, smem);
    if (e != cudaSuccess) return e;
    QkNormArgs m = n;
    long long blocks = 0;
    qk_grid(m, (32 / LPR) * qk_unroll(LPR), per_sm, blocks);
    kern<<<(unsigned)blocks, 32 * kQkWarps, smem, s>>>(m, a);
    return cudaGetLastError();
}

// Sequences of at least this many tokens take two blocks per SM for rows
// of four chunks per lane.
constexpr long long kQkLongT = 16384;

template <typename T, int LPR>
static cudaError_t qk_split_cpl(int cpl, const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    if (cpl == 2) return qk_launch_split<T, LPR, 2, 3>(n, a, s);
    if (n.T >= kQkLongT) return qk_launch_split<T, LPR, 4, 2>(n, a, s);
    return qk_launch_split<T, LPR, 4, 3>(n, a, s);
}

template <typename T>
static cudaError_t qk_dispatch(const QkNormArgs &n, const MropeAngles &a, cudaStream_t s)
{
    constexpr int EC = QkElem<T>::EC;
    // a rotary slice of 4, 8 or 16 lanes and 2 or 4 of its widths per row
    const int lr = 2 * n.half / EC, cpl = n.head_dim / (2 * n.half);
    if (2 * n.half < n.head_dim && n.head_dim % (2 * n.half) == 0 && (cpl == 2 || cpl == 4)) {
        if (lr == 4) return qk_split_cpl<T, 4>(cpl, n, a, s);
        if (lr == 8) return qk_split_cpl<T, 8>(cpl, n, a, s);
        if (lr == 16) return qk_split_cpl<T, 16>(cpl, n, a, s);
    }
    if (2 * n.half == n.head_dim) {
        if (lr == 8) return qk_launch_pair<T, 4>(n, a, s);
        if (lr == 16) return qk_launch_pair<T, 8>(n, a, s);
        if (lr == 32) return qk_launch_pair<T, 16>(n, a, s);
    }
    switch (n.head_dim / EC) {
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
