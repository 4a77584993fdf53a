// Language-model multimodal RoPE kernels: axis map, cos / sin tables, and the
// in-place partial rotate_half rotation (from tables, or fused with the angle
// computation).
//
// "Qwen3-VL" notes (frankmowj.github.io), Qwen3VLTextRotaryEmbedding;
// "Interleaved Rotary Position Embedding" (taking-lying-flat.github.io),
// apply_rotary_pos_emb; "M01 RMSNorm and multimodal RoPE" (kuanzhou.online).
#include <algorithm>

#include <type_traits>

#include "ipe_rotary_tma.cuh"

namespace ipe {

// ------------------------------------------------------------- axis map
__global__ void mrope_axis_map_kernel(int half, int s0, int s1, int s2, int interleaved, int8_t *axis)
{
    const int section[3] = {s0, s1, s2};
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < half; j += gridDim.x * blockDim.x)
        axis[j] = (int8_t)mrope_axis(j, section, interleaved);
}

cudaError_t launch_mrope_axis_map(int half, const int *section, int interleaved, int8_t *axis,
                                  cudaStream_t s)
{
    mrope_axis_map_kernel<<<1, 256, 0, s>>>(half, section[0], section[1], section[2], interleaved, axis);
    return cudaGetLastError();
}

cudaError_t mrope_axis_map_attributes(cudaFuncAttributes *attr)
{
    return cudaFuncGetAttributes(attr, mrope_axis_map_kernel);
}

// ---------------------------------------------------------- cos / sin
// Block (G, 256 / G): threadIdx.x is one of the G = half / V groups of V
// consecutive frequencies of a token, threadIdx.y a token.  Each thread
// takes U tokens per pass (their position loads in flight together) and
// writes both halves of cat(f, f) for cos and sin with V-wide stores.
// Write-stream bound: the 67 MB of tables at rot 64 / T = 131072 take about
// 1.2x the time of a plain fill of the same size.  Measured best: one token
// per pass, six 256-thread blocks per SM, one resident wave.
constexpr int kCsTokens = 1;

template <int V>
__global__ void __launch_bounds__(256, 6) mrope_cos_sin_kernel(const __grid_constant__ MropeAngles a,
                                                                               int half, float *__restrict__ cos_out,
                                                                               float *__restrict__ sin_out)
{
    constexpr int U = kCsTokens;
    const int j0 = threadIdx.x * V;
    int ax[V];
    float inv[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {          // fixed per thread: its frequencies
        ax[e] = mrope_axis(j0 + e, a.section, a.interleaved);
        inv[e] = a.inv[j0 + e];
    }
    const long long stride = (long long)gridDim.x * blockDim.y;
    // positions of the next pass are loaded while this pass computes
    int p0[U], p1[U], p2[U];
    auto load = [&](long long t0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long t = t0 + u * stride;
            if (t < a.T) {
                p0[u] = __ldg(a.positions + t);
                p1[u] = __ldg(a.positions + a.T + t);
                p2[u] = __ldg(a.positions + 2 * a.T + t);
            }
        }
    };
    long long t0 = (long long)blockIdx.x * blockDim.y + threadIdx.y;
    if (t0 < a.T) load(t0);
    for (; t0 < a.T; t0 += U * stride) {
        int q0[U], q1[U], q2[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            q0[u] = p0[u];
            q1[u] = p1[u];
            q2[u] = p2[u];
        }
        if (t0 + U * stride < a.T) load(t0 + U * stride);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long t = t0 + u * stride;
            if (t >= a.T) break;
            Pack<float, V> c, s;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const int pos = ax[e] == 0 ? q0[u] : (ax[e] == 1 ? q1[u] : q2[u]);
                const float angle = __fmul_rn(__int2float_rn(pos), inv[e]);
                sincosf(angle, &s.v[e], &c.v[e]);
            }
            float *co = cos_out + t * 2 * half + j0;
            float *so = sin_out + t * 2 * half + j0;
            st_pack<float, V>(co, c);
            st_pack<float, V>(co + half, c);
            st_pack<float, V>(so, s);
            st_pack<float, V>(so + half, s);
        }
    }
}

template <int V>
static cudaError_t cos_sin_vec(const MropeAngles &a, int half, float *cos_out, float *sin_out, cudaStream_t s)
{
    const int gx = half / V;
    const int gy = std::max(1, 256 / gx);
    const long long need = (a.T + (long long)kCsTokens * gy - 1) / ((long long)kCsTokens * gy);
    // one resident wave: no second, partial wave to wait for at the end
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mrope_cos_sin_kernel<V>, gx * gy, 0);
    if (e != cudaSuccess) return e;
    const int blocks = (int)std::max<long long>(1, std::min(need, (long long)sm_count() * std::max(per_sm, 1)));
    mrope_cos_sin_kernel<V><<<blocks, dim3(gx, gy), 0, s>>>(a, half, cos_out, sin_out);
    return cudaGetLastError();
}

cudaError_t launch_mrope_cos_sin(const MropeAngles &a, int half, float *cos_out, float *sin_out,
                                 cudaStream_t s)
{
    const bool v4 = half % 4 == 0 && (uintptr_t)cos_out % 16 == 0 && (uintptr_t)sin_out % 16 == 0;
    return v4 ? cos_sin_vec<4>(a, half, cos_out, sin_out, s) : cos_sin_vec<1>(a, half, cos_out, sin_out, s);
}

// Widest vector (elements) that divides half, head_dim and both strides and
// that both base pointers are aligned to.
int pick_vec(const RotArgs &r, int elem_bytes)
{
    const int max_vec = 16 / elem_bytes;
    for (int v = max_vec; v > 1; v >>= 1) {
        const uintptr_t align = (uintptr_t)v * elem_bytes;
        if (r.half % v || r.head_dim % v || r.q_stride % v || r.k_stride % v) continue;
        if (r.q && ((uintptr_t)r.q % align)) continue;
        if (r.k && ((uintptr_t)r.k % align)) continue;
        return v;
    }
    return 1;
}

// VEC >= 2 always holds on the TMA path (16-byte rotary rows and strides).
template <typename T, class Src>
static cudaError_t dispatch_tma(const TmaRotArgs &t, const RotArgs &r, const Src &src, cudaStream_t s)
{
    const int v = pick_vec(r, sizeof(T));
    if constexpr (sizeof(T) == 2) {
        if (v == 8) return launch_rotary_tma_vec<T, 8, Src>(t, src, s);
    }
    if (v >= 4) return launch_rotary_tma_vec<T, 4, Src>(t, src, s);
    return launch_rotary_tma_vec<T, 2, Src>(t, src, s);
}

// HF rounding mode (hf): the same engines with cos / sin cast to the
// activation dtype and each product and sum rounded to it.
template <typename T, bool HF>
using MropeTmaOf = std::conditional_t<HF, HfTmaSrc<MropeTmaSrc, T>, MropeTmaSrc>;
template <typename T, bool HF>
using TableTmaOf = std::conditional_t<HF, HfTmaSrc<TableTmaSrc, T>, TableTmaSrc>;
template <typename T, bool HF>
using MropeVecOf = std::conditional_t<HF, HfVecSrc<MropeSrc, T>, MropeSrc>;
template <typename T, bool HF>
using TableVecOf = std::conditional_t<HF, HfVecSrc<TableSrc, T>, TableSrc>;

// Head split for the TMA ring: tokens whose rotary rows are too wide for a
// ring of 8-row tiles at two blocks per SM (Qwen3-Omni: 36 heads x 128
// channels = 9 KB) are rotated as two rows of half the heads each, when q
// and k are contiguous per token and their head counts are even: the same
// memory viewed as [2T, H/2, D].  Two consumer warps then share a token and
// the angle source maps each row back to its token; the ring runs two
// stages at two blocks per SM instead of one block per SM.  Measured on
// B200 (Omni, T = 32768): the fused MRoPE 107.6 -> 101.2 us.  (The table
// rotation, at 0.93 of the copy rate unsplit, measured slower split.)
static bool head_split(const RotArgs &r, int eb, RotArgs &h)
{
    const long long row_bytes = (long long)(r.hq + r.hk) * 2 * r.half * eb;
    if (row_bytes * kTmaRows <= 36864 || r.hq % 2 || r.hk % 2) return false;
    if ((r.hq && r.q_stride != (long long)r.hq * r.head_dim) || (r.hk && r.k_stride != (long long)r.hk * r.head_dim))
        return false;
    h = r;
    h.rows = 2 * r.rows;
    h.hq = r.hq / 2;
    h.hk = r.hk / 2;
    h.q_stride = (long long)h.hq * r.head_dim;
    h.k_stride = (long long)h.hk * r.head_dim;
    return true;
}

template <typename T, bool HF>
static cudaError_t rotary_mrope(const RotArgs &r0, const MropeAngles &a0, cudaStream_t s)
{
    RotArgs r = r0;
    MropeAngles a = a0;
    RotArgs hs;
    if (head_split(r0, sizeof(T), hs)) {
        r = hs;
        a.row_shift = 1;
    }
    TmaRotArgs t;
    if (tma_rot_args(r, sizeof(T), t)) {
        // positions [3, T] as a {T, 3} tensor: rows must be 16-byte multiples;
        // a tile of P rows holds P >> row_shift tokens
        const uint64_t dims[2] = {(uint64_t)a.T, 3};
        const uint64_t str[1] = {(uint64_t)a.T * 4};
        const uint32_t box[2] = {(uint32_t)(t.P >> a.row_shift), 3};
        t.aux_tma = a.T % 4 == 0 && encode_tmap(&t.taux0, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, a.positions, dims, str, box);
        t.aux_bytes = (unsigned)(t.P >> a.row_shift) * 3 * 4;
        MropeTmaOf<T, HF> src{MropeTmaSrc{a}};
        return dispatch_tma<T>(t, r, src, s);
    }
    r = r0;
    a = a0;
    MropeVecOf<T, HF> src{MropeSrc{a}};
    return dispatch_vec<T>(r, src, s);
}

cudaError_t launch_rotary_mrope(bool bf16, const RotArgs &r, const MropeAngles &a, cudaStream_t s, bool hf)
{
    if (hf) return bf16 ? rotary_mrope<__nv_bfloat16, true>(r, a, s) : rotary_mrope<float, true>(r, a, s);
    return bf16 ? rotary_mrope<__nv_bfloat16, false>(r, a, s) : rotary_mrope<float, false>(r, a, s);
}

template <typename T, bool HF>
static cudaError_t rotary_table(const RotArgs &r, const TableAngles &a, cudaStream_t s)
{
    // (no head split: on the Omni rows it measured 104.5 -> 106.6 us)
    TmaRotArgs t;
    if (tma_rot_args(r, sizeof(T), t)) {
        const int rot = 2 * r.half;
        const uint64_t dims[2] = {(uint64_t)rot, (uint64_t)r.rows};
        const uint64_t str[1] = {(uint64_t)rot * 4};
        const uint32_t box[2] = {(uint32_t)rot, (uint32_t)t.P};
        t.aux_tma = encode_tmap(&t.taux0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.cos, dims, str, box) &&
                    encode_tmap(&t.taux1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.sin, dims, str, box);
        t.aux_bytes = 2u * t.P * rot * 4;
        TableTmaOf<T, HF> src{TableTmaSrc{a}};
        return dispatch_tma<T>(t, r, src, s);
    }
    TableVecOf<T, HF> src{TableSrc{a}};
    return dispatch_vec<T>(r, src, s);
}

cudaError_t launch_rotary_table(bool bf16, const RotArgs &r, const TableAngles &a, cudaStream_t s, bool hf)
{
    if (hf) return bf16 ? rotary_table<__nv_bfloat16, true>(r, a, s) : rotary_table<float, true>(r, a, s);
    return bf16 ? rotary_table<__nv_bfloat16, false>(r, a, s) : rotary_table<float, false>(r, a, s);
}

}  // namespace ipe
