// One generation step of the language model's positional encoding: for each
// sequence of the batch one new token, whose position is recovered from its
// sequence index and the rope delta saved at prefill, then (optionally) the
// QK-RMSNorm, the rotation of q and k, and the write of the rotated k and of
// v into their KV-cache slots -- one launch.
//
// "Interleaved Rotary Position Embedding" (taking-lying-flat.github.io),
// compute_3d_position_ids(): after prefill the position of a token is its
// sequence index plus the sample's delta, the same on all three axes, so the
// interleaved / chunked axis map no longer matters and every frequency takes
// the angle fl32(fl32(p) * inv_freq[j]).  The follow-up questions of the
// "M01 RMSNorm and multimodal RoPE (interleaved / chunked)" drill ask how
// decode should compute the cos / sin of its single new token: here the lanes
// that hold rotary chunks compute them in registers, and they are never stored.
//
// Work is split finer than in the prefill kernel: a warp takes one token and
// a small group of its head rows (q rows, then k rows, then v rows when a
// cache is written), so a batch of a few dozen tokens still spreads over
// every SM.
#include "ipe_chunk.cuh"

namespace ipe {

constexpr int kDecWarps = 4;          // 128-thread blocks
constexpr int kDecUnroll = 2;         // head rows per lane in flight
constexpr unsigned kDecBadPosition = 21;   // seq_pos + delta outside [0, 2^24)
constexpr unsigned kDecBadSlot = 22;       // a cache slot at or beyond num_slots

template <typename T, int LPR, bool NORM>
__global__ void __launch_bounds__(32 * kDecWarps) mrope_decode_kernel(const __grid_constant__ DecodeArgs d,
                                                                     const __grid_constant__ MropeAngles a,
                                                                     long long num_slots)
{
    constexpr int EC = QkElem<T>::EC;
    constexpr int NP = EC / 2;
    constexpr int RPW = 32 / LPR;
    constexpr int GROUP = RPW * kDecUnroll;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = d.half, rot = 2 * half, D = d.head_dim;
    const int c = lane % LPR, sub = lane / LPR, e0 = c * EC;
    const bool rotary = e0 < rot, first_half = e0 < half;
    const int j0 = first_half ? e0 : e0 - half;
    const int partner = rotary ? (first_half ? lane + half / EC : lane - half / EC) : lane;
    const int HQK = d.hq + d.hk;
    const int H = HQK + (d.v_cache ? d.hk : 0);     // q rows, k rows, then v rows
    const int groups = (H + GROUP - 1) / GROUP;
    const long long item = (long long)blockIdx.x * kDecWarps + warp;
    const long long t = item / groups;
    if (t >= d.B) return;                           // the whole warp leaves
    const int h0 = (int)(item % groups) * GROUP;

    // this lane's chunk of row h of token t (q, k or v)
    auto row_ptr = [&](int h) -> const T * {
        if (h < d.hq) return static_cast<const T *>(d.q) + t * d.q_stride + (long long)h * D + e0;
        if (h < HQK) return static_cast<const T *>(d.k) + t * d.k_stride + (long long)(h - d.hq) * D + e0;
        return static_cast<const T *>(d.v) + t * d.v_stride + (long long)(h - HQK) * D + e0;
    };
    Pack<uint32_t, 4> x[kDecUnroll];
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
        const int h = h0 + u * RPW + sub;
        if (h < H) {
            x[u] = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(row_ptr(h)));
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) x[u].v[i] = 0u;
        }
    }

    // position of the new token, the same on all three axes
    const long long p = (long long)d.seq_pos[t] + (d.deltas ? d.deltas[t] : 0);
    if ((p < 0 || p >= (1LL << 24)) && h0 == 0 && lane == 0) record_fault(d.status, kDecBadPosition);
    const float fp = __ll2float_rn(p);
    float2 co[NP], si[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        co[i] = make_float2(1.f, 1.f);
        si[i] = make_float2(0.f, 0.f);
        if (rotary) {
            float s0, c0, s1, c1;
            sincosf(__fmul_rn(fp, a.inv[j0 + 2 * i]), &s0, &c0);
            sincosf(__fmul_rn(fp, a.inv[j0 + 2 * i + 1]), &s1, &c1);
            co[i] = make_float2(c0, c1);
            si[i] = first_half ? make_float2(-s0, -s1) : make_float2(s0, s1);
        }
    }
    long long slot = d.slots ? d.slots[t] : -1;
    if (slot >= num_slots) {
        if (h0 == 0 && lane == 0) record_fault(d.status, kDecBadSlot);
        slot = -1;
    }
    Pack<uint32_t, 4> wq, wk;
    if constexpr (NORM) {
        wq = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(static_cast<const T *>(d.q_weight) + e0));
        wk = ld_pack<uint32_t, 4>(reinterpret_cast<const uint32_t *>(static_cast<const T *>(d.k_weight) + e0));
    }
    const float inv_d = __frcp_rn((float)D);   // exact: D is a power of two

#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
        // every lane takes part in the shuffles; rows past H are zeros, never stored
        const int h = h0 + u * RPW + sub;
        const bool is_q = h < d.hq, is_v = h >= HQK;
        Pack<uint32_t, 4> y = x[u];
        if constexpr (NORM) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = is_q ? wq.v[i] : wk.v[i];
            const Pack<uint32_t, 4> yn = rms_norm_chunk<T, LPR>(x[u], w, inv_d, d.eps);
            if (!is_v) y = yn;
        }
        Pack<uint32_t, 4> o = rotate_row_chunk<T>(y, co, si, partner);
        if (is_v) o = y;
        if (h >= H) continue;
        if (!is_v) st_pack<uint32_t, 4>(reinterpret_cast<uint32_t *>(const_cast<T *>(row_ptr(h))), o);
        if (slot >= 0 && !is_q) {
            T *cache = static_cast<T *>(is_v ? d.v_cache : d.k_cache) + slot * d.cache_stride +
                       (long long)(h - (is_v ? HQK : d.hq)) * D + e0;
            st_pack<uint32_t, 4>(reinterpret_cast<uint32_t *>(cache), o);
        }
    }
}

template <typename T, int LPR>
static cudaError_t decode_launch(const DecodeArgs &d, const MropeAngles &a, long long num_slots, cudaStream_t s)
{
    constexpr int GROUP = (32 / LPR) * kDecUnroll;
    const int H = d.hq + d.hk + (d.v_cache ? d.hk : 0);
    const long long items = d.B * ((H + GROUP - 1) / GROUP);
    const long long blocks = (items + kDecWarps - 1) / kDecWarps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (d.q_weight)
        mrope_decode_kernel<T, LPR, true><<<(unsigned)blocks, 32 * kDecWarps, 0, s>>>(d, a, num_slots);
    else
        mrope_decode_kernel<T, LPR, false><<<(unsigned)blocks, 32 * kDecWarps, 0, s>>>(d, a, num_slots);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t decode_dispatch(const DecodeArgs &d, const MropeAngles &a, long long num_slots, cudaStream_t s)
{
    switch (d.head_dim / QkElem<T>::EC) {
    case 32: return decode_launch<T, 32>(d, a, num_slots, s);
    case 16: return decode_launch<T, 16>(d, a, num_slots, s);
    case 8: return decode_launch<T, 8>(d, a, num_slots, s);
    case 4: return decode_launch<T, 4>(d, a, num_slots, s);
    case 2: return decode_launch<T, 2>(d, a, num_slots, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_mrope_decode(bool bf16, const DecodeArgs &d, const MropeAngles &a, long long num_slots,
                                cudaStream_t s)
{
    return bf16 ? decode_dispatch<__nv_bfloat16>(d, a, num_slots, s) : decode_dispatch<float>(d, a, num_slots, s);
}

}  // namespace ipe
