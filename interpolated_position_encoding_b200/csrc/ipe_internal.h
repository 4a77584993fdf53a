// Internal descriptors and launchers shared by the C ABI (ipe_api.cu) and the
// kernels.  Host-validated: every launcher assumes its arguments passed the
// checks in ipe_api.cu.
#pragma once

#include <cstdint>

#include <cuda.h>            // CUtensorMap (types only; the encoder is resolved at run time)
#include <cuda_runtime.h>

namespace ipe {

// ---------------------------------------------------------------- vision
// One image of a vision call: its (t, h, w) grid, the first merge-row strip
// it owns among all images, and its first output row (cu_seqlens offset).
struct VisImage {
    int t, h, w;
    int strip0;
    long long row0;
};

// Descriptor passed by value as a kernel parameter.  MAXIMG is 16 for small
// calls (a 400-byte parameter block) and 1024 otherwise.
template <int MAXIMG>
struct VisDesc {
    int n_images;
    int merge;
    int grid_side;
    int n_strips;        // sum over images of h / merge
    long long n_patch;   // sum over images of t h w
    VisImage img[MAXIMG];
};

// The first MAXIMG images of a descriptor (MAXIMG = 16: a 400-byte kernel
// parameter block instead of about 25 KB, for calls of at most 16 images).
template <int MAXIMG>
inline VisDesc<MAXIMG> shrink(const VisDesc<1024> &d)
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

// Interpolation output / table of one call.
struct InterpArgs {
    const void *table;   // [G*G, hidden]
    void *out;           // [n_patch, hidden]
    int hidden;
    int n_slices;        // channel slices of the interpolation grid
};

// ---------------------------------------------------------------- rotary
// In-place rotation of the first 2*half channels of every head row.
struct RotArgs {
    void *q, *k;
    long long rows;        // tokens or patches
    long long q_stride, k_stride;   // elements between consecutive rows
    int hq, hk, head_dim;
    int half;              // rot_dim / 2
    int rows_per_tile;
};

constexpr int kMaxHalf = 256;
constexpr int kMaxVisFreq = 64;    // head_dim / 4 of the vision rotary

// Angle sources of the rotation kernels (kernel parameters).
struct MropeAngles {               // angle = fl32(pos[axis(j)]) * inv[j]
    const int32_t *positions;      // [3, T]
    long long T;
    int section[3];
    int interleaved;
    float inv[kMaxHalf];
    int row_shift = 0;             // rotary rows per token = 1 << row_shift (the TMA ring's head split)
};

struct TableAngles {               // cos / sin read from [T, 2*half] tables
    const float *cos;
    const float *sin;
};

struct VisAngleFreqs {             // vision 2-D angles: row * inv[i], col * inv[i]
    int nf;                        // frequencies per axis (= head_dim / 4)
    float inv[kMaxVisFreq];
};

// ------------------------------------------------------- TMA rotation path
// In-place rotation fed by tiled TMA loads and drained by TMA stores (see
// ipe_rotary_tma.cuh).  Each tile is P rows, one per consumer warp.  A stage
// holds P q-row slots and P k-row slots (each 128-byte aligned, the rotary
// slice of every head of one row), then the aux boxes.
struct TmaRotArgs {
    CUtensorMap tq, tk;      // [rows, heads, head_dim] -> box {rot, heads, P}  (whole-tile loads)
    CUtensorMap tq1, tk1;    // same tensors, box {rot, heads, 1}             (per-row loads, stores)
    CUtensorMap taux0;       // positions [3, T] -> box {P, 3}, or cos [T, rot] -> box {rot, P}
    CUtensorMap taux1;       // sin [T, rot] -> box {rot, P}
    long long rows;
    int hq, hk, half;
    int P;                   // rows per tile = consumer warps
    int stages;
    int aux_tma;             // 1 when taux0 (and taux1) are loaded by TMA
    int dense_q, dense_k;    // 1: one box per tile (slot = row bytes, a multiple of 128)
    int lane_rows;           // 1: lane i rotates head row i (<= 32 rows); 0: lanes sweep chunks
    int swap_shift;          // lanes with bit `swap_shift` set read the second half first
    unsigned slot_q, slot_k; // bytes of one row slot
    unsigned stage_bytes, off_k, off_aux0, off_aux1;
    unsigned row_bytes_q, row_bytes_k, aux_bytes;
    long long wait_limit;    // SM cycles before a barrier wait gives up
    long long skip_tile;     // test hook: the producer never loads this tile (-1: none)
    unsigned *status;        // fault word (ipe_device_status)
};

// ----------------------------------------------- fused QK-RMSNorm + MRoPE
struct QkNormArgs {
    void *q, *k;                      // [T, hq, D], [T, hk, D], rewritten in place
    const void *q_weight, *k_weight;  // [D] norm weights, activation dtype
    long long T;
    long long q_stride, k_stride;
    int hq, hk, head_dim, half, half_pad;
    float eps;
    int groups, rows_per_item;        // a token's head rows split over `groups` warps (set by the launcher)
};

cudaError_t launch_qk_norm_mrope(bool bf16, const QkNormArgs &n, const MropeAngles &a, cudaStream_t s);

// One generation step (ipe_mrope_decode): per sequence one new token whose
// position is seq_pos + delta on all three axes; optional QK-RMSNorm; q and k
// rotated in place; k (rotated) and v written to their cache slots.
struct DecodeArgs {
    void *q, *k;                      // [B, hq, D], [B, hk, D], rewritten in place
    const void *v;                    // [B, hk, D] or NULL
    void *k_cache, *v_cache;          // rows of [hk, D] at slot * cache_stride, or NULL
    const int64_t *slots;             // [B] cache slot of each new token (< 0: none) or NULL
    const int32_t *seq_pos;           // [B] sequence index of the new token
    const int32_t *deltas;            // [B] rope deltas or NULL
    const void *q_weight, *k_weight;  // [D] norm weights, or both NULL (no norm)
    long long B;
    long long q_stride, k_stride, v_stride, cache_stride;   // elements
    int hq, hk, head_dim, half;
    float eps;
    unsigned *status;
};

cudaError_t launch_mrope_decode(bool bf16, const DecodeArgs &d, const MropeAngles &a, long long num_slots,
                                cudaStream_t s);

// ------------------------------------------------------- position table
// Tile of the position-table kernels: 256 threads x 4 consecutive slots.
constexpr int kRiThreads = 256;
constexpr int kRiPer = 4;
constexpr int kRiTile = kRiThreads * kRiPer;

// One call of ipe_mrope_rope_index, validated on the host.  The workspace
// carries the per-tile aggregates, the per-tile carries, one record per sample
// and the grid prefix sums, each at a 256-byte aligned offset.
struct RopeIndexArgs {
    const void *types, *mask;          // [B, L] of id_bytes each; mask may be NULL
    const void *img_grid, *vid_grid;   // [n, 3] of grid_bytes each
    int id_bytes, grid_bytes;
    long long B, L;
    int tiles_per_row;                 // ceil(L / kRiTile)
    int n_img, n_vid, merge;
    int32_t *pos;                      // [3, B, L]
    int32_t *deltas;                   // [B]
    void *agg, *state, *sample;        // workspace sections: per tile counts and states, per sample records
    unsigned *flags;                   // [B * tiles_per_row] publication flag of each tile
    unsigned *ticket;                  // next tile to hand out
    long long *img_adv;                // [n_img + 1] prefix of the image advances
    long long *vid_slices, *vid_adv;   // [n_vid + 1] prefixes of slices and of slice advances
    unsigned *status;
    long long wait_limit;              // SM cycles before a look-back wait gives up
    long long skip_tile;               // test hook: this tile never publishes (-1: none)
};

// Bytes of each workspace section for a call; the sum is the workspace size.
struct RopeIndexLayout {
    size_t agg, state, flags, sample, ticket, img_adv, vid_slices, vid_adv, total;
};
RopeIndexLayout rope_index_layout(long long B, long long L, int n_img, int n_vid);
cudaError_t launch_rope_index(const RopeIndexArgs &a, cudaStream_t s);

// Test hooks and the device status word (ipe_api.cu).
unsigned *device_status_word();
long long debug_skip_tile();
long long debug_wait_limit();

// TMA rotation arguments for the q / k of `r` (tensor maps, strides, test
// hooks, status word).  False when the shapes, strides or alignment do not
// allow tiled TMA (the caller then uses the vector-load path).
bool tma_rot_args(const RotArgs &r, int elem_bytes, TmaRotArgs &t);

// Tiled tensor map over `base` (rank <= 3, dims inner first, strides in bytes
// for dims 1..rank-1).  False if the driver rejects it.
bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides, const uint32_t *box);

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_mrope_cos_sin(const MropeAngles &a, int half, float *cos_out, float *sin_out,
                                 cudaStream_t s);
// Attributes of a library kernel as loaded on the current device (the
// architecture its code was built for).
cudaError_t mrope_axis_map_attributes(cudaFuncAttributes *attr);
cudaError_t launch_mrope_axis_map(int half, const int *section, int interleaved, int8_t *axis,
                                  cudaStream_t s);
cudaError_t launch_rotary_mrope(bool bf16, const RotArgs &r, const MropeAngles &a, cudaStream_t s,
                                bool hf = false);
cudaError_t launch_rotary_table(bool bf16, const RotArgs &r, const TableAngles &a, cudaStream_t s,
                                bool hf = false);

cudaError_t launch_vis_plan(const VisDesc<1024> &d, int32_t *idx4, float *w4, int32_t *rowcol,
                            cudaStream_t s);
// Shared memory of one interpolation block for this request.
size_t vis_interp_block_smem(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia);
cudaError_t launch_vis_interp(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s);
cudaError_t launch_vis_interp_hf(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s);
// `budget`: shared memory per rotary block to aim for (0: the default).
cudaError_t launch_vis_rope(bool bf16, const VisDesc<1024> &d, const RotArgs &r,
                            const VisAngleFreqs &f, cudaStream_t s, size_t budget = 0);

// Widest vector (elements, <= 16 bytes) that divides half, head_dim and both
// strides of `r` and that both base pointers are aligned to.
int pick_vec(const RotArgs &r, int elem_bytes);

// Shared-memory bytes of one interpolation block covering `slices` 128-byte
// channel slices (the host checks the limit at one slice).
size_t interp_smem_bytes(bool bf16, int merge, int grid_side, int slices = 1);

}  // namespace ipe
