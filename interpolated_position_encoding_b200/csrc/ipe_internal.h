// Internal descriptors and launchers shared by the C ABI (ipe_api.cu) and the
// kernels.  Host-validated: every launcher assumes its arguments passed the
// checks in ipe_api.cu.
#pragma once

#include <cstdint>

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
};

struct TableAngles {               // cos / sin read from [T, 2*half] tables
    const float *cos;
    const float *sin;
};

struct VisAngleFreqs {             // vision 2-D angles: row * inv[i], col * inv[i]
    int nf;                        // frequencies per axis (= head_dim / 4)
    float inv[kMaxVisFreq];
};

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_mrope_cos_sin(const MropeAngles &a, int half, float *cos_out, float *sin_out,
                                 cudaStream_t s);
cudaError_t launch_mrope_axis_map(int half, const int *section, int interleaved, int8_t *axis,
                                  cudaStream_t s);
cudaError_t launch_rotary_mrope(bool bf16, const RotArgs &r, const MropeAngles &a, cudaStream_t s);
cudaError_t launch_rotary_table(bool bf16, const RotArgs &r, const TableAngles &a, cudaStream_t s);

cudaError_t launch_vis_plan(const VisDesc<1024> &d, int32_t *idx4, float *w4, int32_t *rowcol,
                            cudaStream_t s);
cudaError_t launch_vis_interp(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, cudaStream_t s);
cudaError_t launch_vis_rope(bool bf16, const VisDesc<1024> &d, const RotArgs &r,
                            const VisAngleFreqs &f, cudaStream_t s);
cudaError_t launch_vis_fused(bool bf16, const VisDesc<1024> &d, const InterpArgs &ia, const RotArgs &r,
                             const VisAngleFreqs &f, cudaStream_t s);

// Widest vector (elements, <= 16 bytes) that divides half, head_dim and both
// strides of `r` and that both base pointers are aligned to.
int pick_vec(const RotArgs &r, int elem_bytes);

// Shared-memory bytes of one interpolation block (host check of the limit).
size_t interp_smem_bytes(bool bf16, int merge, int grid_side);

}  // namespace ipe
