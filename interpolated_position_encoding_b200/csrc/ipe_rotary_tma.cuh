// TMA-fed in-place rotation (sm_100a).
//
// Warp 0 is the producer: one lane streams tiles of P rows (tokens or
// patches) from HBM into a ring of shared-memory stages with tiled TMA loads
// (cp.async.bulk.tensor over [rows, heads, head_dim] with boxes of
// {rot, heads, *}, so only the rotary slice of each head row moves), keeping
// up to `stages` tiles in flight.  Warps 1..P are consumers, one row of the
// tile each: the warp computes the row's (cos, sin) once into its own
// shared-memory slot (one sincosf per frequency, shared by every head of q and
// k), rotates the row's head rows in place in shared memory, and a TMA store
// writes the row back; once the store has read the slot the warp frees the
// stage (one row later, when the ring has three or more stages).  No
// block-wide barrier runs inside the loop.
//
// Every wait is bounded (TmaRotArgs::wait_limit cycles): a warp that gives up
// records a fault in the status word and raises a shared abort flag, the
// others leave their loops, and the producer waits (bounded) for the loads it
// still has in flight before the block exits.
#pragma once

#include "ipe_rotary.cuh"
#include "ipe_tma.cuh"

namespace ipe {

constexpr int kTmaConsumers = 8;
constexpr int kTmaRows = kTmaConsumers;             // rows per tile: one per consumer warp
constexpr int kTmaThreads = 32 * (1 + kTmaConsumers);
constexpr int kTmaMaxStages = 8;
// Two blocks per SM.  Measured on the fused MRoPE of the large prefill:
// 112 KB (three 28.8 KB stages) 0.85 of the copy peak, 72 KB (three blocks
// of two stages) 0.82, 220 KB (one block of seven stages) 0.58.
constexpr size_t kTmaBlockSmem = 112 * 1024;

__host__ __device__ inline unsigned align128(unsigned v) { return (v + 127u) & ~127u; }

// (cos, sin) slot of one consumer warp, in floats: cos [half], sin [half],
// -sin [half] (4 floats further, so sin and -sin chunks fall in different
// banks) and, for tables whose halves may differ, cos_hi [half], sin_hi [half].
struct CsSlot {
    float *c, *s, *ns, *ch, *sh;
};

__host__ __device__ inline size_t tma_cs_floats(int half, bool hi) { return (size_t)half * (hi ? 5 : 3) + (hi ? 8 : 4); }

// Packed fp32 pairs (sm_100a): two independent correctly rounded operations.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// VEC elements <-> VEC/2 fp32 pairs (element 2i in .x, 2i+1 in .y).
template <typename T, int VEC>
__device__ __forceinline__ void load_pairs(const T *p, float2 *v)
{
    if constexpr (sizeof(T) == 2) {
        const Pack<uint32_t, VEC / 2> w = ld_pack<uint32_t, VEC / 2>(reinterpret_cast<const uint32_t *>(p));
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i)
            v[i] = make_float2(__uint_as_float(w.v[i] << 16), __uint_as_float(w.v[i] & 0xffff0000u));
    } else {
        const Pack<float2, VEC / 2> f = ld_pack<float2, VEC / 2>(reinterpret_cast<const float2 *>(p));
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i) v[i] = f.v[i];
    }
}

template <typename T, int VEC>
__device__ __forceinline__ void store_pairs(T *p, const float2 *v)
{
    if constexpr (sizeof(T) == 2) {
        Pack<uint32_t, VEC / 2> w;
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(v[i].x, v[i].y);   // one rounding each
            w.v[i] = *reinterpret_cast<const uint32_t *>(&b);
        }
        st_pack<uint32_t, VEC / 2>(reinterpret_cast<uint32_t *>(p), w);
    } else {
        Pack<float2, VEC / 2> f;
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i) f.v[i] = v[i];
        st_pack<float2, VEC / 2>(reinterpret_cast<float2 *>(p), f);
    }
}

template <int VEC>
__device__ __forceinline__ void load_coef(const float *p, float2 *v)
{
    const Pack<float2, VEC / 2> f = ld_pack<float2, VEC / 2>(reinterpret_cast<const float2 *>(p));
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) v[i] = f.v[i];
}

// ------------------------------------------------------------ angle sources
// angles(): (cos, sin) of every frequency of tile row c (global row `row`)
// into the warp's slot.  issue_aux(): TMA loads of per-tile side data.
// Sources with kEarlyAngles also offer angles_early(), the same values for
// frequencies lane + 32 i computed into registers from global memory only
// (so a warp can work out its next row's while that row's stage is still
// loading), and angles_store(), which writes them to the slot.

constexpr int kEarlyRounds = 4;   // half <= 128 on the TMA path
struct AngleRegs {
    float c[kEarlyRounds], s[kEarlyRounds];
};

__device__ __forceinline__ void store_angle_regs(const TmaRotArgs &r, int lane, const CsSlot &cs, const AngleRegs &g)
{
#pragma unroll
    for (int i = 0; i < kEarlyRounds; ++i) {
        const int j = lane + 32 * i;
        if (j < r.half) {
            cs.c[j] = g.c[i];
            cs.s[j] = g.s[i];
            cs.ns[j] = -g.s[i];
        }
    }
}

struct MropeTmaSrc {
    static constexpr bool kHi = false;
    static constexpr bool kHf = false;
    static constexpr bool kTwoBlockBound = true;
    // early angles would read the positions from global memory on the
    // row's critical path instead of from the stage: slower (the large
    // prefill 162.6 -> 164 us, Omni 107.6 -> 118 us)
    static constexpr bool kEarlyAngles = false;
    MropeAngles a;
    __device__ __forceinline__ void issue_aux(const TmaRotArgs &r, uint32_t stage, int r0, uint32_t bar) const
    {
        tma_load_2d(stage + r.off_aux0, &r.taux0, r0 >> a.row_shift, 0, bar);   // positions [3, P >> row_shift]
    }
    // position on axis ax of the token of tile row c (global row `row`):
    // from the stage when the positions came with it, else from memory
    __device__ __forceinline__ int pos_of(const TmaRotArgs &r, const unsigned char *stage, int c, long long row,
                                          int ax) const
    {
        const int32_t *spos = reinterpret_cast<const int32_t *>(stage + r.off_aux0);
        return r.aux_tma ? spos[ax * (r.P >> a.row_shift) + (c >> a.row_shift)]
                         : __ldg(a.positions + (long long)ax * a.T + (row >> a.row_shift));
    }
    // `round` maps each cos / sin value before it is stored (the HF mode
    // rounds to the activation dtype here, in the one write of the slot)
    template <class Round>
    __device__ __forceinline__ void angles_rounded(const TmaRotArgs &r, const unsigned char *stage, int c,
                                                   long long row, int lane, const CsSlot &cs, Round round) const
    {
        for (int j = lane; j < r.half; j += 32) {
            const int pos = pos_of(r, stage, c, row, mrope_axis(j, a.section, a.interleaved));
            // fl32(fl32(pos) * inv_freq[j]): one rounded product, no contraction
            const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
            float sn, cn;
            sincosf(angle, &sn, &cn);
            sn = round(sn);
            cs.c[j] = round(cn);
            cs.s[j] = sn;
            cs.ns[j] = -sn;
        }
    }
    __device__ __forceinline__ void angles(const TmaRotArgs &r, const unsigned char *stage, int c, long long row,
                                           int lane, const CsSlot &cs) const
    {
        angles_rounded(r, stage, c, row, lane, cs, [](float v) { return v; });
    }
    // HF mode, bf16: cos, sin and -sin rounded to bf16 and stored as bf16x2
    // words of the frequency pairs (2i, 2i+1), word i at the front of each
    // array; lane j takes frequency j and its odd neighbour's values by
    // shuffle, so the slot is written once.  -sin flips the sign bit (exact).
    __device__ __forceinline__ void angles_bf16_words(const TmaRotArgs &r, const unsigned char *stage, int c,
                                                      long long row, int lane, const CsSlot &cs) const
    {
        for (int j0 = 0; j0 < r.half; j0 += 32) {   // every lane takes part in the shuffles
            const int j = j0 + lane;
            float sn = 0.f, cn = 0.f;
            if (j < r.half) {
                const int pos = pos_of(r, stage, c, row, mrope_axis(j, a.section, a.interleaved));
                const float angle = __fmul_rn(__int2float_rn(pos), a.inv[j]);
                sincosf(angle, &sn, &cn);
            }
            const uint32_t cb = __bfloat16_as_ushort(__float2bfloat16_rn(cn));
            const uint32_t sb = __bfloat16_as_ushort(__float2bfloat16_rn(sn));
            const uint32_t cb1 = __shfl_down_sync(0xffffffffu, cb, 1), sb1 = __shfl_down_sync(0xffffffffu, sb, 1);
            if (!(lane & 1) && j < r.half) {
                const int i = j >> 1;
                reinterpret_cast<uint32_t *>(cs.c)[i] = cb | (cb1 << 16);
                reinterpret_cast<uint32_t *>(cs.s)[i] = sb | (sb1 << 16);
                reinterpret_cast<uint32_t *>(cs.ns)[i] = (sb ^ 0x8000u) | ((sb1 ^ 0x8000u) << 16);
            }
        }
    }
};

struct TableTmaSrc {
    static constexpr bool kHi = true;
    static constexpr bool kHf = false;
    static constexpr bool kTwoBlockBound = false;
    static constexpr bool kEarlyAngles = false;
    TableAngles a;
    __device__ __forceinline__ void issue_aux(const TmaRotArgs &r, uint32_t stage, int r0, uint32_t bar) const
    {
        tma_load_2d(stage + r.off_aux0, &r.taux0, 0, r0, bar);      // cos [P, rot]
        tma_load_2d(stage + r.off_aux1, &r.taux1, 0, r0, bar);      // sin [P, rot]
    }
    __device__ __forceinline__ void angles(const TmaRotArgs &r, const unsigned char *stage, int c, long long row,
                                           int lane, const CsSlot &cs) const
    {
        const int half = r.half, rot = 2 * half;
        const float *sc = r.aux_tma ? reinterpret_cast<const float *>(stage + r.off_aux0) + (size_t)c * rot
                                    : a.cos + row * rot;
        const float *ss = r.aux_tma ? reinterpret_cast<const float *>(stage + r.off_aux1) + (size_t)c * rot
                                    : a.sin + row * rot;
        for (int j = lane; j < half; j += 32) {
            cs.c[j] = sc[j];
            cs.s[j] = ss[j];
            cs.ns[j] = -ss[j];
            cs.ch[j] = sc[j + half];
            cs.sh[j] = ss[j + half];
        }
    }
};

template <int MAXIMG>
struct VisTmaSrc {
    static constexpr bool kHi = false;
    static constexpr bool kHf = false;
    static constexpr bool kTwoBlockBound = true;
    // the angles need only the row index: worked out a row ahead (the
    // one-call vision pair 67.2 -> 65.9 us on the batch of 8 and 127.1 ->
    // 125.3 us on the video; the rotary alone on the video 103.1 -> 104.2 us)
    static constexpr bool kEarlyAngles = true;
    VisDesc<MAXIMG> d;
    VisAngleFreqs f;
    __device__ __forceinline__ void angles_early(const TmaRotArgs &r, long long row, int lane, AngleRegs &g) const
    {
        int prow, pcol;
        patch_row_col(d, row, prow, pcol);
        const int nf = f.nf;
#pragma unroll
        for (int i = 0; i < kEarlyRounds; ++i) {
            const int j = lane + 32 * i;
            if (j < r.half) {
                // angles [row * inv (nf) | col * inv (nf)]
                const int v = j < nf ? prow : pcol;
                sincosf(__fmul_rn(__int2float_rn(v), f.inv[j < nf ? j : j - nf]), &g.s[i], &g.c[i]);
            }
        }
    }
    __device__ __forceinline__ void angles_store(const TmaRotArgs &r, int lane, const CsSlot &cs,
                                                 const AngleRegs &g) const
    {
        store_angle_regs(r, lane, cs, g);
    }
    __device__ __forceinline__ void issue_aux(const TmaRotArgs &, uint32_t, int, uint32_t) const {}
};

// HF rounding mode of a source: its cos / sin cast to the activation dtype T
// before they are used (each lane rounds the entries it wrote).
template <class Base, typename T>
struct HfTmaSrc : Base {
    static constexpr bool kHf = true;
    static constexpr bool kEarlyAngles = false;
    __device__ __forceinline__ void angles(const TmaRotArgs &r, const unsigned char *stage, int c, long long row,
                                           int lane, const CsSlot &cs) const
    {
        if constexpr (!Base::kHi) {
            // the fused MRoPE rounds as it writes the slot (bf16: as words)
            if constexpr (sizeof(T) == 2)
                Base::angles_bf16_words(r, stage, c, row, lane, cs);
            else
                Base::angles_rounded(r, stage, c, row, lane, cs, [](float v) { return round_to_dtype<T>(v); });
            return;
        }
        Base::angles(r, stage, c, row, lane, cs);
        for (int j = lane; j < r.half; j += 32) {
            const float sn = round_to_dtype<T>(cs.s[j]);
            cs.c[j] = round_to_dtype<T>(cs.c[j]);
            cs.s[j] = sn;
            cs.ns[j] = -sn;
            if constexpr (Base::kHi) {
                cs.ch[j] = round_to_dtype<T>(cs.ch[j]);
                cs.sh[j] = round_to_dtype<T>(cs.sh[j]);
            }
        }
        if constexpr (sizeof(T) == 2 && Base::kHi) {
            // bf16 tables: the pairs (2i, 2i+1) of every array as bf16x2
            // words at the front of that array (exact: the values are bf16
            // already), read that way by every chunk's packed products; each
            // round of 32 words is read in full before any of it is written.
            // Measured on B200 (large prefill): the HF table rotation 178.1
            // -> 171.7 us.  (The fused MRoPE packs as it writes instead: a
            // second pass over its three arrays cost more than it saved.)
            float *arr[5] = {cs.c, cs.s, cs.ns, cs.ch, cs.sh};
            constexpr int NA = 5;
            const int nw = r.half / 2;
            for (int i0 = 0; i0 < nw; i0 += 32) {
                const int i = i0 + lane;
                uint32_t w[NA];
                __syncwarp();
#pragma unroll
                for (int q = 0; q < NA; ++q) {
                    w[q] = 0u;
                    if (i < nw) {
                        const __nv_bfloat162 b = __floats2bfloat162_rn(arr[q][2 * i], arr[q][2 * i + 1]);
                        w[q] = *reinterpret_cast<const uint32_t *>(&b);
                    }
                }
                __syncwarp();
                if (i < nw) {
#pragma unroll
                    for (int q = 0; q < NA; ++q) reinterpret_cast<uint32_t *>(arr[q])[i] = w[q];
                }
            }
        }
    }
};

// HF combine of a pair: each product rounded to T, their sum evaluated in
// fp32 (the caller's store rounds it to T).
template <typename T>
__device__ __forceinline__ float2 hf_pair(float2 a, float2 b)
{
    a = make_float2(round_to_dtype<T>(a.x), round_to_dtype<T>(a.y));
    b = make_float2(round_to_dtype<T>(b.x), round_to_dtype<T>(b.y));
    return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
}

// The coefficients of one chunk: fp32 pairs, or bf16x2 words in the bf16 HF
// mode (the slot holds words there).
template <typename T, int VEC, bool HI, bool HF>
struct RotCoef {
    static constexpr bool kWords = HF && sizeof(T) == 2;
    Pack<uint32_t, VEC / 2> c1w, c2w, s1w, s2w;
    float2 c1[VEC / 2], c2[VEC / 2], s1[VEC / 2], s2[VEC / 2];
};

// Coefficients of chunk u with the lane's swap bit: C1 / S1 for the values
// at the first address, C2 / S2 for the second (see rotate_chunk_with).
template <typename T, int VEC, bool HI, bool HF>
__device__ __forceinline__ void load_rot_coef(const CsSlot &cs, int u, bool swap, RotCoef<T, VEC, HI, HF> &k)
{
    const int o = u * VEC;
    const float *C1 = HI ? (swap ? cs.ch : cs.c) + o : cs.c + o;
    const float *C2 = HI ? (swap ? cs.c : cs.ch) + o : cs.c + o;
    const float *S1 = (swap ? (HI ? cs.sh : cs.s) : cs.ns) + o;
    const float *S2 = (swap ? cs.ns : (HI ? cs.sh : cs.s)) + o;
    if constexpr (RotCoef<T, VEC, HI, HF>::kWords) {
        // word o / 2 of an array holds elements o and o + 1
        auto words = [&](const float *a) {
            return ld_pack<uint32_t, VEC / 2>(reinterpret_cast<const uint32_t *>(a - o) + o / 2);
        };
        k.c1w = words(C1);
        k.s1w = words(S1);
        k.s2w = words(S2);
        k.c2w = HI ? words(C2) : k.c1w;
    } else {
        load_coef<VEC>(C1, k.c1);
        load_coef<VEC>(S1, k.s1);
        load_coef<VEC>(S2, k.s2);
        if constexpr (HI) load_coef<VEC>(C2, k.c2);
    }
}

// One chunk: elements [u VEC, u VEC + VEC) of the first half of head row `p`
// and the matching chunk of the second half, rotated in place with the
// coefficients `k` of that chunk.  With `swap` the lane reads (and writes)
// the second half first, which spreads neighbouring rows over the banks;
// the formula is the same either way:
//   x'[j]     = x[j] cos_j         - x[j+h] sin_j
//   x'[j + h] = x[j + h] cos_{j+h} + x[j] sin_{j+h}
// written as  w1 = v1 C1 + v2 S1,  w2 = v2 C2 + v1 S2  on the values v1, v2
// at the first and second address, with C / S chosen (not computed) per lane.
template <typename T, int VEC, bool HI, bool HF>
__device__ __forceinline__ void rotate_chunk_with(T *p, int half, int u, bool swap, const RotCoef<T, VEC, HI, HF> &k)
{
    static_assert(VEC >= 2, "pairs");
    T *pa = p + u * VEC, *pb = pa + half;
    T *p1 = swap ? pb : pa, *p2 = swap ? pa : pb;
    if constexpr (RotCoef<T, VEC, HI, HF>::kWords) {
        // bf16 HF: every product and the sum as one packed bf16x2 operation
        // each, rounding where the fp32-then-cast steps do (mul_bf16x2 /
        // add_bf16x2).
        using W = Pack<uint32_t, VEC / 2>;
        const W r1 = ld_pack<uint32_t, VEC / 2>(reinterpret_cast<const uint32_t *>(p1));
        const W r2 = ld_pack<uint32_t, VEC / 2>(reinterpret_cast<const uint32_t *>(p2));
        W o1, o2;
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i) {
            o1.v[i] = add_bf16x2(mul_bf16x2(r1.v[i], k.c1w.v[i]), mul_bf16x2(r2.v[i], k.s1w.v[i]));
            o2.v[i] = add_bf16x2(mul_bf16x2(r2.v[i], k.c2w.v[i]), mul_bf16x2(r1.v[i], k.s2w.v[i]));
        }
        st_pack<uint32_t, VEC / 2>(reinterpret_cast<uint32_t *>(p1), o1);
        st_pack<uint32_t, VEC / 2>(reinterpret_cast<uint32_t *>(p2), o2);
        return;
    }
    float2 v1[VEC / 2], v2[VEC / 2], w1[VEC / 2], w2[VEC / 2];
    load_pairs<T, VEC>(p1, v1);
    load_pairs<T, VEC>(p2, v2);
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
        const float2 c2 = HI ? k.c2[i] : k.c1[i];
        if constexpr (HF) {
            w1[i] = hf_pair<T>(mul2(v1[i], k.c1[i]), mul2(v2[i], k.s1[i]));
            w2[i] = hf_pair<T>(mul2(v2[i], c2), mul2(v1[i], k.s2[i]));
        } else {
            w1[i] = fma2(v1[i], k.c1[i], mul2(v2[i], k.s1[i]));
            w2[i] = fma2(v2[i], c2, mul2(v1[i], k.s2[i]));
        }
    }
    store_pairs<T, VEC>(p1, w1);
    store_pairs<T, VEC>(p2, w2);
}

template <typename T, int VEC, bool HI, bool HF>
__device__ __forceinline__ void rotate_chunk(T *p, int half, int u, bool swap, const CsSlot &cs)
{
    RotCoef<T, VEC, HI, HF> k;
    load_rot_coef<T, VEC, HI, HF>(cs, u, swap, k);
    rotate_chunk_with<T, VEC, HI, HF>(p, half, u, swap, k);
}

// Rotate the head rows of one tile row (q slot then k slot) in shared memory.
template <typename T, int VEC, bool HI, bool HF>
__device__ __forceinline__ void rotate_slots(const TmaRotArgs &a, unsigned char *sq, unsigned char *sk, int lane,
                                             const CsSlot &cs)
{
    const int half = a.half, rot = 2 * half, nvec = half / VEC, H = a.hq + a.hk;
    T *q = reinterpret_cast<T *>(sq);
    T *k = reinterpret_cast<T *>(sk);
    if (a.lane_rows) {
        // lane i owns head row i; all lanes read the same (cos, sin) chunk
        if (lane < H) {
            T *p = lane < a.hq ? q + lane * rot : k + (lane - a.hq) * rot;
            const bool swap = (lane >> a.swap_shift) & 1;
            for (int u = 0; u < nvec; ++u) rotate_chunk<T, VEC, HI, HF>(p, half, u, swap, cs);
        }
    } else {
        // lanes sweep (head, chunk) with the chunk fastest; odd heads swap
        int h = lane / nvec, u = lane - h * nvec;
        const int dh = 32 / nvec, du = 32 - dh * nvec;
        if (du == 0 && !(dh & 1)) {
            // the lane keeps its chunk and its swap bit for every head it
            // visits: the chunk's coefficients are read once per row
            const bool swap = h & 1;
            RotCoef<T, VEC, HI, HF> kc;
            load_rot_coef<T, VEC, HI, HF>(cs, u, swap, kc);
            for (; h < H; h += dh) {
                T *p = h < a.hq ? q + h * rot : k + (h - a.hq) * rot;
                rotate_chunk_with<T, VEC, HI, HF>(p, half, u, swap, kc);
            }
            return;
        }
        while (h < H) {
            T *p = h < a.hq ? q + h * rot : k + (h - a.hq) * rot;
            rotate_chunk<T, VEC, HI, HF>(p, half, u, h & 1, cs);
            u += du;
            h += dh;
            if (u >= nvec) {
                u -= nvec;
                ++h;
            }
        }
    }
}

// Shared memory of one block: 128 B alignment slack, the stages, 2 barriers
// per stage, the abort flag (16 B) and the consumers' (cos, sin) slots.
__host__ __device__ inline size_t tma_smem_bytes(const TmaRotArgs &a, bool hi)
{
    const size_t cs = (tma_cs_floats(a.half, hi) * sizeof(float) + 15) & ~size_t(15);
    return 128 + (size_t)a.stages * a.stage_bytes + 16 * (size_t)a.stages + 16 + (size_t)kTmaConsumers * cs;
}

// The whole pipeline of one block over tiles bid, bid + nb, ... (the caller
// passes its dynamic shared memory).
template <typename T, int VEC, class Src>
__device__ __forceinline__ void rotary_tma_block(const TmaRotArgs &a, const Src &src, unsigned char *smem_raw,
                                                 long long bid, long long nb)
{
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
    const int S = a.stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)S * a.stage_bytes);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 2 * S);
    float *slots = reinterpret_cast<float *>(bars + 2 * S + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&bars[s]), 1);                    // full: the producer's expect_tx
            mbar_init(smem_addr(&bars[S + s]), kTmaConsumers);    // empty: one arrival per consumer warp
        }
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const long long ntiles = (a.rows + a.P - 1) / a.P;

    if (warp == 0) {
        if (lane != 0) return;
        // ------------------------------------------------------- producer
        if (a.hq) prefetch_tmap(a.dense_q ? &a.tq : &a.tq1);
        if (a.hk) prefetch_tmap(a.dense_k ? &a.tk : &a.tk1);
        long long last_round[kTmaMaxStages];
        for (int s = 0; s < kTmaMaxStages; ++s) last_round[s] = -1;
        bool aborted = false;
        long long it = 0;
        for (long long tile = bid; tile < ntiles; tile += nb, ++it) {
            const int s = (int)(it % S);
            const long long round = it / S;
            if (!mbar_wait(smem_addr(&bars[S + s]), (uint32_t)((round & 1) ^ 1), a.wait_limit, abort)) {
                if (!*abort) record_fault(a.status, kFaultEmptyWait);
                *abort = 1;
                aborted = true;
                break;
            }
            if (tile == a.skip_tile) continue;    // test hook: this stage never fills
            const uint32_t full = smem_addr(&bars[s]);
            const uint32_t st = smem_addr(smem + (size_t)s * a.stage_bytes);
            const int r0 = (int)(tile * a.P);
            const int valid = (int)min((long long)a.P, a.rows - r0);
            // a whole-tile box counts all P rows (rows past the end are
            // zero-filled); per-row boxes are issued for valid rows only
            const unsigned tx = (a.dense_q ? a.P : valid) * a.row_bytes_q + (a.dense_k ? a.P : valid) * a.row_bytes_k +
                                (a.aux_tma ? a.aux_bytes : 0u);
            mbar_arrive_expect_tx(full, tx);
            if (a.hq) {
                if (a.dense_q) tma_load_3d(st, &a.tq, 0, 0, r0, full);
                else
                    for (int p = 0; p < valid; ++p) tma_load_3d(st + p * a.slot_q, &a.tq1, 0, 0, r0 + p, full);
            }
            if (a.hk) {
                if (a.dense_k) tma_load_3d(st + a.off_k, &a.tk, 0, 0, r0, full);
                else
                    for (int p = 0; p < valid; ++p)
                        tma_load_3d(st + a.off_k + p * a.slot_k, &a.tk1, 0, 0, r0 + p, full);
            }
            if (a.aux_tma) src.issue_aux(a, st, r0, full);
            last_round[s] = round;
        }
        if (aborted || *abort) {
            // loads still in flight must land before the block releases its memory
            for (int s = 0; s < S; ++s)
                if (last_round[s] >= 0 &&
                    !mbar_wait(smem_addr(&bars[s]), (uint32_t)(last_round[s] & 1), a.wait_limit, nullptr))
                    record_fault(a.status, kFaultDrainWait);
        }
        return;
    }

    // ----------------------------------------------------------- consumers
    const int c = warp - 1;
    const size_t cs_stride = (tma_cs_floats(a.half, Src::kHi) + 3) & ~size_t(3);
    CsSlot cs;
    cs.c = slots + (size_t)c * cs_stride;
    cs.s = cs.c + a.half;
    cs.ns = cs.s + a.half + 4;
    cs.ch = Src::kHi ? cs.ns + a.half + 4 : cs.c;
    cs.sh = Src::kHi ? cs.ch + a.half : cs.s;
    // With three or more stages a warp frees each stage one row late: after
    // committing row r's store it waits only until row r-1's store has read
    // its slot (wait_group.read 1) and frees that stage, so each store's read
    // of shared memory overlaps the next row's wait and arithmetic.  With two
    // stages that would leave one in flight, so the warp waits for its own
    // store and frees the stage at once.  Measured on B200: the fused MRoPE
    // of the large prefill (three stages) 169.9 -> 161.6 us; rows of 9 KB
    // (two stages) 125 us at once against 191 us one row late.
    const bool late = S >= 3;
    int pending = -1;   // stage whose row store may still be reading it
    long long it = 0;
    // Sources with kEarlyAngles: a warp works out its next row's (cos, sin)
    // into registers while its current row's store reads the stage and the
    // next stage loads, then only writes them to its slot.
    AngleRegs ang;
    if constexpr (Src::kEarlyAngles) {
        if (bid < ntiles && bid * a.P + c < a.rows) src.angles_early(a, bid * a.P + c, lane, ang);
    }
    for (long long tile = bid; tile < ntiles; tile += nb, ++it) {
        const int s = (int)(it % S);
        bool ok = mbar_wait(smem_addr(&bars[s]), (uint32_t)((it / S) & 1), a.wait_limit, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            if (lane == 0) {
                if (!*abort) record_fault(a.status, kFaultFullWait);
                *abort = 1;
            }
            break;
        }
        unsigned char *stage = smem + (size_t)s * a.stage_bytes;
        const long long row = tile * a.P + c;
        if (row < a.rows) {
            unsigned char *sq = stage + (size_t)c * a.slot_q;
            unsigned char *sk = stage + a.off_k + (size_t)c * a.slot_k;
            if constexpr (Src::kEarlyAngles)
                src.angles_store(a, lane, cs, ang);
            else
                src.angles(a, stage, c, row, lane, cs);
            __syncwarp();
            rotate_slots<T, VEC, Src::kHi, Src::kHf>(a, sq, sk, lane, cs);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (a.hq) tma_store_3d(&a.tq1, smem_addr(sq), 0, 0, (int)row);
                if (a.hk) tma_store_3d(&a.tk1, smem_addr(sk), 0, 0, (int)row);
            }
        }
        __syncwarp();
        if (lane == 0) {
            bulk_commit();   // this row's store (an empty group past the last row)
            // a slot may be refilled once the store has read it
            if (!late) {
                bulk_wait_read_all();
                mbar_arrive(smem_addr(&bars[S + s]));
            } else if (pending >= 0) {
                bulk_wait_read_1();
                mbar_arrive(smem_addr(&bars[S + pending]));
            }
        }
        pending = s;
        if constexpr (Src::kEarlyAngles) {
            // the next row's angles, after the stage release
            const long long nrow = (tile + nb) * a.P + c;
            if (tile + nb < ntiles && nrow < a.rows) src.angles_early(a, nrow, lane, ang);
        }
    }
    if (lane == 0) bulk_wait_all();
}

// Launch bounds by angle source (Src::kTwoBlockBound).  With two blocks per
// SM as the bound ptxas gives the consumers up to 113 registers (88-96 for
// bf16 rows), against 66-96 with the thread count alone.  Measured on B200:
// HF fused MRoPE 165.4 -> 161.2 us, Qwen3-Omni MRoPE 121.1 -> 118.1 us, the
// one-call vision pair 129.7 -> 127.2 us (video) and 71.5 -> 68.7 us (batch
// of 8), the vision rotary on the batch of 8 47.0 -> 45.1 us and on the video
// unchanged (102 us), the fused MRoPE unchanged; the table rotation slower
// (Omni 119.2 -> 128.3 us), so table sources keep the thread count alone.
template <typename T, int VEC, class Src>
__global__ void __launch_bounds__(kTmaThreads, 2) rotary_tma_kernel(const __grid_constant__ TmaRotArgs a,
                                                                    const __grid_constant__ Src src)
{
    extern __shared__ unsigned char smem_raw[];
    rotary_tma_block<T, VEC, Src>(a, src, smem_raw, blockIdx.x, gridDim.x);
}

template <typename T, int VEC, class Src>
__global__ void __launch_bounds__(kTmaThreads) rotary_tma_kernel_tb(const __grid_constant__ TmaRotArgs a,
                                                                    const __grid_constant__ Src src)
{
    extern __shared__ unsigned char smem_raw[];
    rotary_tma_block<T, VEC, Src>(a, src, smem_raw, blockIdx.x, gridDim.x);
}

template <typename T, int VEC, class Src>
constexpr auto rotary_tma_entry()
{
    if constexpr (Src::kTwoBlockBound)
        return &rotary_tma_kernel<T, VEC, Src>;
    else
        return &rotary_tma_kernel_tb<T, VEC, Src>;
}

// --------------------------------------------------------------- launch
// Lanes with bit `shift` of their index set read the second half first; the
// shift with the fewest shared-memory bank conflicts for lane-per-row access
// (row stride, half offset and access width in bytes).
inline int best_swap_shift(unsigned row_bytes, unsigned half_bytes, unsigned access_bytes)
{
    int best = 3, best_cost = 1 << 30;
    const unsigned lanes_per_wave = access_bytes >= 16 ? 8 : access_bytes == 8 ? 16 : 32;
    for (int shift = 1; shift <= 4; ++shift) {
        int cost = 0;
        for (unsigned w0 = 0; w0 < 32; w0 += lanes_per_wave) {
            int load[32] = {0};
            for (unsigned l = w0; l < w0 + lanes_per_wave; ++l) {
                const unsigned off = l * row_bytes + (((l >> shift) & 1) ? half_bytes : 0);
                for (unsigned b = 0; b < access_bytes; b += 4) ++load[((off + b) / 4) % 32];
            }
            int worst = 0;
            for (int b = 0; b < 32; ++b) worst = load[b] > worst ? load[b] : worst;
            cost += worst;
        }
        if (cost < best_cost) {
            best_cost = cost;
            best = shift;
        }
    }
    return best;
}

// Fills the stage layout of `a` and picks the stage count for the
// shared-memory budget: the deepest ring within `first` bytes (a caller
// that shares the SMs with another kernel passes less than the default)
// when two stages fit there, else as below.
template <typename T, int VEC, class Src>
void tma_layout(TmaRotArgs &a, size_t first = kTmaBlockSmem)
{
    const unsigned eb = sizeof(T);
    const unsigned rot = 2u * a.half;
    a.row_bytes_q = a.hq * rot * eb;
    a.row_bytes_k = a.hk * rot * eb;
    a.dense_q = a.row_bytes_q % 128 == 0;
    a.dense_k = a.row_bytes_k % 128 == 0;
    a.slot_q = align128(a.row_bytes_q);
    a.slot_k = align128(a.row_bytes_k);
    a.off_k = a.P * a.slot_q;
    a.off_aux0 = a.off_k + a.P * a.slot_k;
    const unsigned aux0 = a.aux_tma ? a.aux_bytes - (Src::kHi ? a.aux_bytes / 2 : 0) : 0;
    a.off_aux1 = a.off_aux0 + align128(aux0);
    a.stage_bytes = a.off_aux1 + align128(a.aux_tma && Src::kHi ? a.aux_bytes / 2 : 0);
    const int H = a.hq + a.hk;
    a.lane_rows = H <= 32 && (rot * eb) % 128 != 0;
    a.swap_shift = best_swap_shift(rot * eb, a.half * eb, VEC * eb);
    // deepest ring within ~112 KB (two blocks per SM); rows too wide for two
    // stages there get up to ~220 KB (one block per SM)
    for (size_t budget : {first, kTmaBlockSmem, size_t(220 * 1024)}) {
        a.stages = 2;
        for (int st = kTmaMaxStages; st >= 2; --st) {
            a.stages = st;
            if (tma_smem_bytes(a, Src::kHi) <= budget) break;
        }
        if (tma_smem_bytes(a, Src::kHi) <= budget) break;
    }
}

// Lays out `a` and launches the pipeline on the SMs.
template <typename T, int VEC, class Src>
cudaError_t launch_rotary_tma_vec(TmaRotArgs a, const Src &src, cudaStream_t s, size_t first = kTmaBlockSmem)
{
    tma_layout<T, VEC, Src>(a, first);
    const size_t smem = tma_smem_bytes(a, Src::kHi);
    auto kern = rotary_tma_entry<T, VEC, Src>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTmaThreads, smem);
    if (e != cudaSuccess) return e;
    const long long ntiles = (a.rows + a.P - 1) / a.P;
    const long long cap = (long long)sm_count() * std::max(per_sm, 1);
    const int blocks = (int)std::max<long long>(1, std::min(ntiles, cap));
    kern<<<blocks, kTmaThreads, smem, s>>>(a, src);
    return cudaGetLastError();
}

}  // namespace ipe
