/*
 * ipe.h -- C ABI of the B200 (sm_100a) interpolated-position-encoding library
 * (libipe.so): the positional-encoding hot path of Qwen3-VL / Qwen3.5-style
 * vision-language models.
 *
 *   vision tower   vis_pos_interp      bilinear 48x48 position table -> patch grid, 2x2 merge order
 *                  vis_rope2d          2-D (row, col) rotary over the whole head
 *                  vis_pos_interp_rope2d  both in one call (two kernels, concurrent)
 *   language model rope_inv_freq       default RoPE inverse frequencies (host)
 *                  mrope_axis_map      per-frequency T/H/W axis (interleaved or chunked)
 *                  mrope_cos_sin       multimodal cos / sin tables
 *                  apply_rotary_partial  rotate_half rotation of the first rot_dim channels
 *                  mrope_apply         the three above fused; cos / sin never leave registers
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Return value: an ipe_status.  On anything but IPE_OK, ipe_last_error()
 *   returns a message for the calling thread, and nothing was launched unless
 *   the status is IPE_ECUDA from the launch itself.
 * - Every check happens on the host before any launch: sizes, divisibility,
 *   alignment of vectorised pointers and strides, and that each device pointer
 *   is device memory of the current device whose allocation covers the bytes
 *   the call touches.  Kernels never trap or assert.
 * - Device pointers are caller-owned.  The library allocates no memory and
 *   keeps no pointer after it returns.  Small host arrays (grid_thw, section,
 *   inv_freq) are copied by value into kernel parameters before the call
 *   returns, so the caller may reuse them at once.
 * - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *   legacy default stream) of the current device.
 * - Rotations are in place.  vis_pos_interp and mrope_cos_sin write separate
 *   outputs.  Two calls that touch the same memory on different streams race.
 * - Element counts and strides are in elements, not bytes.
 * - Floating-point arithmetic is fp32; bf16 results are rounded once (to
 *   nearest even) at the end.  sin / cos are CUDA's accurate sincosf.
 * - CUDA graphs: the device entry points can be captured into a graph and
 *   replayed.  Make one call of each before the capture: a first call may
 *   create the library's per-device stream and events and look up driver
 *   entry points, which must not happen inside a capture.
 *
 * Pages cited (title -- section):
 *   [QVL]  "Qwen3-VL" notes, frankmowj.github.io
 *   [IRPE] "Interleaved Rotary Position Embedding", taking-lying-flat.github.io
 *   [M01]  "M01 RMSNorm and multimodal RoPE (interleaved / chunked)", kuanzhou.online
 *   [VLM]  "VLM", llm.rainlin.net
 *   [CRT]  cortiq-engine 0.8.52 src/qwen3vis.rs, docs.rs
 */
#ifndef IPE_H
#define IPE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { IPE_F32 = 0, IPE_BF16 = 1 } ipe_dtype;

typedef enum {
    IPE_OK = 0,
    IPE_EINVAL = 1,  /* a size, count or pointer the operation does not accept  */
    IPE_EALIGN = 2,  /* a pointer or stride breaks the vector alignment        */
    IPE_ELIMIT = 3,  /* above a documented library limit (images, dims, T)     */
    IPE_ECUDA = 4,   /* a CUDA runtime call or the launch failed               */
    IPE_EDEVICE = 5  /* a kernel gave up a bounded wait (ipe_device_status)    */
} ipe_status;

/* Library limits (IPE_ELIMIT above them). */
#define IPE_MAX_IMAGES 1024     /* images per vision call                     */
#define IPE_MAX_HALF 256        /* rot_dim / 2 of the text rotary             */
#define IPE_MAX_POSITION 16777216 /* positions must lie in [0, 2^24): fl32(pos) is exact */
#define IPE_MAX_GRIDS 16384     /* image grids, and video grids, per position-table call */

/* Message for the last non-OK status returned on this thread ("" if none). */
const char *ipe_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int ipe_version(void);

/* ---------------------------------------------------------------------------
 * ipe_kernel_arch -- the compute capability a library kernel was compiled
 * for, as the CUDA runtime loaded it on the current device
 * (cudaFuncGetAttributes: binaryVersion and ptxVersion, major * 10 + minor;
 * 100 for sm_100a).  Needs a CUDA device; IPE_ECUDA when the library's code
 * cannot run on it.  No counterpart on the pages: it reports which GPU
 * architecture the library's kernels were compiled for.
 *   binary_version, ptx_version   host int*, written.
 * ------------------------------------------------------------------------- */
int ipe_kernel_arch(int *binary_version, int *ptx_version);

/* ---------------------------------------------------------------------------
 * ipe_device_status -- failure report of the kernels that ran on the current
 * device.  The TMA-fed rotation kernels wait on shared-memory barriers; every
 * such wait gives up after a time limit (about one second), records a fault
 * code in a device status word and lets the kernel return instead of spinning.
 * This call synchronises `stream`, reads and clears that word, and returns
 * IPE_OK, or IPE_EDEVICE with a message naming the wait that gave up (the
 * results of the failed launch are then incomplete).  The position-table
 * scan's waits are bounded the same way (code 23).  ipe_mrope_rope_index
 * and ipe_mrope_decode report inputs that only the device can see the same
 * way (codes 16 .. 22, listed there).  Not part of any page: failure
 * reporting of this library.
 * ------------------------------------------------------------------------- */
int ipe_device_status(void *stream);

/* ---------------------------------------------------------------------------
 * ipe_debug_inject -- test hook for the failure path above.  From the next
 * launch on, the producer of the TMA rotation kernels skips the loads of tile
 * `skip_tile` (-1: none), so the consumers waiting for it give up after
 * `wait_cycles` SM clock cycles (0: the default limit); in the position-table
 * scan (ipe_mrope_rope_index) tile `skip_tile` publishes nothing, so the
 * tiles after it give up their look-back the same way.  Host state, not
 * thread-safe; reset with ipe_debug_inject(-1, 0).
 * ------------------------------------------------------------------------- */
int ipe_debug_inject(int64_t skip_tile, int64_t wait_cycles);

/* ---------------------------------------------------------------------------
 * ipe_rope_inv_freq -- default RoPE inverse frequencies, on the host.
 * [IRPE] compute_default_rope_parameters; [M01] problem summary:
 *   inv_freq[j] = 1 / theta^(2j / rot_dim),  j = 0 .. rot_dim/2 - 1
 * with rot_dim = int(head_dim * partial_rotary_factor).  Computed in double,
 * rounded once to fp32.
 *   rot_dim        even, 2 .. 2*IPE_MAX_HALF
 *   theta          > 0 (rope_theta: 1e7 for Qwen3.5 text, 1e6 Qwen3-Omni, 1e4 vision)
 *   inv_freq_host  host array of rot_dim/2 floats, written.
 * ------------------------------------------------------------------------- */
int ipe_rope_inv_freq(int rot_dim, double theta, float *inv_freq_host);

/* ---------------------------------------------------------------------------
 * ipe_mrope_axis_map -- axis (0 = T, 1 = H, 2 = W) of each of the `half`
 * frequencies, written on the device by the same device code the rotary
 * kernels use.
 * Interleaved ([QVL] apply_interleaved_mrope; [M01] problem summary): H where
 * j % 3 == 1 and j < 3*section[1]; W where j % 3 == 2 and j < 3*section[2];
 * T elsewhere.  Chunked ([M01] step-by-step figure, Qwen2-VL / Qwen2.5-Omni):
 * T for j < section[0], H for j < section[0] + section[1], W after.
 *   half        1 .. IPE_MAX_HALF
 *   section     host int32[3] = mrope_section (s_t, s_h, s_w), each >= 0, sum == half
 *   interleaved 1 for interleaved (Qwen3-VL / Qwen3.5 / Qwen3-Omni), 0 for chunked
 *   axis_dev    device int8[half], written.
 * ------------------------------------------------------------------------- */
int ipe_mrope_axis_map(int half, const int32_t *section, int interleaved, int8_t *axis_dev,
                       void *stream);

/* ---------------------------------------------------------------------------
 * ipe_mrope_cos_sin -- multimodal RoPE cos / sin tables.
 * [QVL] Qwen3VLTextRotaryEmbedding.forward; [M01] shape trace rows 2-7:
 *   angle[t, j] = fl32(fl32(positions[axis(j), t]) * inv_freq[j])
 *   cos[t, j] = cos[t, j + half] = cos(angle[t, j]); likewise sin
 * (emb = cat(f, f); attention_scaling = 1).  Kept in fp32 (no cast to the
 * activation dtype).
 *   positions      device int32 [3, T] row-major (rows t, h, w; row stride T),
 *                  values in [0, IPE_MAX_POSITION) (precondition, not checked
 *                  on the device)
 *   T              tokens, >= 0 (T = B*L for a batch of B sequences of length L)
 *   inv_freq_host  host float[half]
 *   half           rot_dim / 2, 1 .. IPE_MAX_HALF
 *   section, interleaved  as for ipe_mrope_axis_map
 *   cos_out, sin_out  device float [T, 2*half] row-major, written.
 * ------------------------------------------------------------------------- */
int ipe_mrope_cos_sin(const int32_t *positions, int64_t T, const float *inv_freq_host, int half,
                      const int32_t *section, int interleaved, float *cos_out, float *sin_out,
                      void *stream);

/* ---------------------------------------------------------------------------
 * ipe_apply_rotary_partial -- rotate_half rotation of the first rot_dim
 * channels of every head of Q and K, in place; channels >= rot_dim untouched.
 * [IRPE] rotate_half / apply_rotary_pos_emb (partial rotary); [M01] L1 hints:
 *   h = rot_dim/2; for j < h:
 *   x'[j]     = x[j] * cos[t, j]         - x[j + h] * sin[t, j]
 *   x'[j + h] = x[j + h] * cos[t, j + h] + x[j] * sin[t, j + h]
 * cos / sin are shared by all heads of a token.
 *   q, k          device, dtype, token-major [T, hq, head_dim] / [T, hk, head_dim];
 *                 heads contiguous (head stride = head_dim); token strides
 *                 q_tok_stride, k_tok_stride (>= heads * head_dim).  k may be
 *                 NULL iff hk == 0, q NULL iff hq == 0.
 *   dtype         IPE_BF16 or IPE_F32
 *   rot_dim       even, 2 .. min(head_dim, 2*IPE_MAX_HALF)
 *   cos, sin      device float [T, rot_dim] row-major (e.g. from ipe_mrope_cos_sin)
 * Vector alignment: accesses are as wide as rot_dim/2, head_dim, the strides
 * and the pointers allow (up to 16 bytes); no alignment is required.
 * ------------------------------------------------------------------------- */
int ipe_apply_rotary_partial(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk,
                             int head_dim, int64_t q_tok_stride, int64_t k_tok_stride,
                             const float *cos, const float *sin, int rot_dim, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_mrope_apply -- ipe_mrope_cos_sin followed by ipe_apply_rotary_partial in
 * one pass: each (token, frequency) angle and its sincosf are computed once
 * and shared by all hq + hk heads; cos / sin are never written to memory.
 * Same arguments and results as the two calls it replaces, with
 * rot_dim = 2 * half.
 * ------------------------------------------------------------------------- */
int ipe_mrope_apply(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                    int64_t q_tok_stride, int64_t k_tok_stride, const int32_t *positions,
                    const float *inv_freq_host, int rot_dim, const int32_t *section,
                    int interleaved, void *stream);

/* ---------------------------------------------------------------------------
 * HF rounding mode of the text rotation: ipe_apply_rotary_partial_hf and
 * ipe_mrope_apply_hf take the same arguments as the calls without the
 * suffix and round where the reference listings round, so that results
 * match those checkpoints' own code bit for bit:
 * [QVL] Qwen3VLTextRotaryEmbedding.forward returns cos / sin cast to the
 * activation dtype; [IRPE] apply_rotary_pos_emb computes
 * (q_rot * cos) + (rotate_half(q_rot) * sin) in that dtype; [M01] hints
 * (cos / sin cast first, then multiplied):
 *   c = dtype(cos), s = dtype(sin)          (fp32 cos / sin as in the default mode)
 *   out = dtype(fl32(dtype(x c) + dtype(rotate_half(x) s)))
 * For fp32 activations every product and the sum are separate fp32
 * roundings (no fused multiply-add).  Pass-through channels are untouched.
 * ------------------------------------------------------------------------- */
int ipe_apply_rotary_partial_hf(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk,
                                int head_dim, int64_t q_tok_stride, int64_t k_tok_stride,
                                const float *cos, const float *sin, int rot_dim, void *stream);
int ipe_mrope_apply_hf(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                       int64_t q_tok_stride, int64_t k_tok_stride, const int32_t *positions,
                       const float *inv_freq_host, int rot_dim, const int32_t *section,
                       int interleaved, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_qk_norm_mrope -- RMSNorm of every head row of Q and K followed by the
 * multimodal rotation of ipe_mrope_apply, in one pass, in place.
 * [M01] problem summary and hints (rms_norm; the vllm-omni note on fusing it
 * with the rotary); [IRPE] RoPE section ("projection and Q norm done" before
 * the rotation):
 *   xn = x * rsqrt(mean(x^2) + eps)      fp32, mean over the head_dim channels
 *   y  = dtype(dtype(xn) * weight)       cast back to the dtype, then the weight
 *   out = y rotated as ipe_mrope_apply (first rot_dim channels); channels
 *         >= rot_dim are y.  All head_dim channels are written.
 * q_weight / k_weight: device [head_dim], dtype (the q_norm / k_norm weights).
 * head_dim: 16-byte chunks per row a power of two in 2 .. 32 (bf16: 16 .. 256,
 * fp32: 8 .. 128); rot_dim / 2 a multiple of 8 (bf16) or 4 (fp32); q, k,
 * weights and token strides 16-byte aligned (IPE_EALIGN otherwise).
 * eps >= 0.  Other arguments as ipe_mrope_apply.
 * ------------------------------------------------------------------------- */
int ipe_qk_norm_mrope(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                      int64_t q_tok_stride, int64_t k_tok_stride, const void *q_weight,
                      const void *k_weight, float eps, const int32_t *positions,
                      const float *inv_freq_host, int rot_dim, const int32_t *section,
                      int interleaved, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_mrope_decode -- one generation step: for each of B sequences one new
 * token, its position recovered from the sequence index and the rope delta,
 * optional QK-RMSNorm, q and k rotated in place, and the rotated k and v
 * written to their KV-cache slots, in one launch.
 * [IRPE] compute_3d_position_ids() ("recovering the positions": sequence
 * index, expanded to three rows, plus the sample's delta); [M01] follow-up
 * questions (decode cos / sin of a single token):
 *   p[b] = seq_pos[b] + rope_deltas[b]      the same on all three axes, so the
 *                                           axis layout (section) plays no part
 *   angle[j] = fl32(fl32(p) * inv_freq[j]); rotation as ipe_mrope_apply
 * seq_pos is the new token's sequence index: cumsum(attention_mask)[-1] - 1
 * with a padding mask, else the cache length before the token.
 *   q, k        device, dtype, [B, hq, head_dim] / [B, hk, head_dim], token
 *               strides q_tok_stride / k_tok_stride (elements), rewritten in place
 *   v           device [B, hk, head_dim], token stride v_tok_stride; read only
 *               when v_cache is given (else may be NULL)
 *   seq_pos     device int32 [B]; rope_deltas device int32 [B] or NULL (0)
 *   q_weight, k_weight  device [head_dim] of dtype, or both NULL: no norm;
 *               with them every q / k row is RMS-normalised first, as
 *               ipe_qk_norm_mrope (eps >= 0)
 *   k_cache, v_cache  device rows of [hk, head_dim] at slot * cache_slot_stride
 *               (elements), num_slots slots; v_cache may be NULL
 *   slot_mapping  device int64 [B]: cache slot of each new token, < 0 = no
 *               write (padding); NULL: no cache write (then both caches NULL)
 * head_dim, rot_dim and alignment as ipe_qk_norm_mrope (q, k, v, caches,
 * weights and all strides 16-byte aligned).  Reported through
 * ipe_device_status: 21 a position outside [0, 2^24); 22 a slot at or beyond
 * num_slots (that write is skipped).
 * ------------------------------------------------------------------------- */
int ipe_mrope_decode(void *q, void *k, const void *v, ipe_dtype dtype, int64_t B, int hq, int hk, int head_dim,
                     int64_t q_tok_stride, int64_t k_tok_stride, int64_t v_tok_stride, const int32_t *seq_pos,
                     const int32_t *rope_deltas, const void *q_weight, const void *k_weight, float eps,
                     const float *inv_freq_host, int rot_dim, void *k_cache, void *v_cache,
                     int64_t cache_slot_stride, int64_t num_slots, const int64_t *slot_mapping, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_mrope_rope_index -- three-axis position table and rope deltas of a batch
 * of B mixed sequences padded to L slots, on the device (no host sync).
 * [IRPE] get_rope_index(): preparing the grids, filtering padding and
 * splitting runs, advancing the position, flattening the vision grid, joining
 * the sequence back, returning positions and deltas; the worked single-batch
 * table; mm_tokens (type codes).  The rules:
 *   - video grid rows (t, h, w) count as t grids (1, h, w), one per temporal
 *     slice; image grids are used as given (llm_t = t);
 *   - one image and one video grid sequence serve the whole batch, consumed
 *     in the order of samples and, within a sample, of appearance;
 *   - per sample the slots with mask 0 are dropped; the kept slots form runs
 *     of equal type; a position starting at 0 walks the runs: a text run
 *     (type 0, or 3 = audio, laid out like text) takes consecutive positions
 *     on all three rows; a vision run (1 image, 2 video) takes the next grid
 *     of its kind and gives its k-th slot, k = (tt*(h/m) + row)*(w/m) + col,
 *     the coordinates (start + tt, start + row, start + col); the position
 *     then moves on by max(h, w) / m;
 *   - dropped slots get 0 on all rows; rope_deltas[b] = (largest coordinate
 *     of the sample) + 1 - (its kept slots), 0 for a sample with none.
 *   mm_token_type_ids  device [B, L] integers of id_bytes (4 or 8) each
 *   attention_mask     device [B, L] of id_bytes, non-zero = kept; NULL keeps all
 *   image_grid_thw     device [n_images, 3] integers of grid_bytes (4 or 8)
 *   video_grid_thw     device [n_videos, 3] of grid_bytes; NULL iff n_videos == 0
 *                      (likewise the image grids)
 *   spatial_merge      m, 1 .. 64
 *   position_ids       device int32 [3, B, L], written (rows t, h, w)
 *   rope_deltas        device int32 [B], written
 *   workspace          device scratch of at least
 *                      ipe_mrope_rope_index_workspace(B, L, n_images, n_videos)
 *                      bytes, 16-byte aligned; overwritten; no initial value
 *                      needed.  Calls that share it must not overlap.
 * Limits: B * L <= 2^31 - 1, L <= 2^30, n_images and n_videos <= IPE_MAX_GRIDS.
 * What only the device sees is reported through ipe_device_status: 16 a
 * vision run found no grid left; 17 a vision run's length differs from its
 * grid's cell count (the pages' listing only fails when a sample's totals
 * differ; here every run is checked); 18 a kept slot of a type other than
 * 0 .. 3 (laid out as text); 19 a grid with t, h or w outside 1 .. 32768;
 * 20 a coordinate beyond the int32 range; 23 a tile of the scan gave up
 * waiting (about a second) for an earlier tile's counts (the table and the
 * deltas are then incomplete).  Otherwise the table is written regardless.
 * Runs on `stream` as a memset of the workspace's tile flags and sample
 * records, then one kernel: a single-pass scan over tiles of 1024 slots.
 * ------------------------------------------------------------------------- */
int ipe_mrope_rope_index(const void *mm_token_type_ids, const void *attention_mask, int id_bytes,
                         int64_t B, int64_t L, const void *image_grid_thw, int n_images,
                         const void *video_grid_thw, int n_videos, int grid_bytes, int spatial_merge,
                         int32_t *position_ids, int32_t *rope_deltas, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Workspace bytes ipe_mrope_rope_index needs for these sizes (0 on bad sizes). */
size_t ipe_mrope_rope_index_workspace(int64_t B, int64_t L, int n_images, int n_videos);

/* ---------------------------------------------------------------------------
 * ipe_mrope_rope_index_static -- ipe_mrope_rope_index for callers that cannot
 * supply device memory at call time (a serving loop that reserved all device
 * memory up front and allows no allocation on its hot path, or a C host
 * program without a device allocator).  No counterpart on the pages: this is
 * an interface choice of this library, the computation is that of
 * ipe_mrope_rope_index.
 * Instead of a caller workspace it uses a scratch array of
 * IPE_ROPE_INDEX_STATIC_BYTES compiled into the library, one per device; the
 * call allocates no memory.  Sizes whose workspace
 * (ipe_mrope_rope_index_workspace) exceeds that are rejected with IPE_ELIMIT.
 * The first call on each device looks the array's address up (with that
 * device current) and so does the set-up work: make it before any stream
 * capture.  After a device reset in the same process the next call on that
 * device finds the remembered address stale and does the set-up again.  The
 * call itself first clears what must start at zero (a memset on `stream`),
 * so the caller clears nothing between calls.  All calls on
 * one device share the array: calls whose kernels overlap in time (on other
 * streams or from other host threads) race.  Arguments and results as
 * ipe_mrope_rope_index without workspace / workspace_bytes.
 * ------------------------------------------------------------------------- */
#define IPE_ROPE_INDEX_STATIC_BYTES (4u << 20) /* 4 MiB: B * L up to about 40 million slots */
int ipe_mrope_rope_index_static(const void *mm_token_type_ids, const void *attention_mask, int id_bytes,
                                int64_t B, int64_t L, const void *image_grid_thw, int n_images,
                                const void *video_grid_thw, int n_videos, int grid_bytes, int spatial_merge,
                                int32_t *position_ids, int32_t *rope_deltas, void *stream);

/* ---------------------------------------------------------------------------
 * Vision grids.  grid_thw_host is a host int32 [n_images, 3] array of
 * (t, h, w) patch grids BEFORE the spatial merge ([VLM] 1.1 Patch; [IRPE]
 * get_rope_index); h and w must be multiples of `merge` (spatial_merge_size,
 * 2 in Qwen3-VL).  Patches of all images are concatenated in grid_thw order
 * (image i starts at row sum_{j<i} t_j h_j w_j, its cu_seqlens offset); within
 * an image, frame-major, then merge-block row, merge-block column, and the
 * merge x merge patches of a block row-major ([QVL] fast_pos_embed_interpolate
 * permute(0, 1, 3, 2, 4, 5); [CRT] positions()).
 * ------------------------------------------------------------------------- */

/* ---------------------------------------------------------------------------
 * ipe_vis_interp_plan -- corner ids, weights and (row, col) of every patch in
 * output order, written by the device code of the interpolation kernels.
 * [QVL] fast_pos_embed_interpolate: sample y = row (G-1)/(h-1) (0 when h = 1),
 * y0 = floor(y), y1 = min(y0 + 1, G-1), dy = y - y0 (likewise x); corners
 * TL, TR, BL, BR = (y0 G + x0, y0 G + x1, y1 G + x0, y1 G + x1), weights
 * ((1-dy)(1-dx), (1-dy)dx, dy(1-dx), dy dx).  Corners use integer arithmetic
 * (y0 = row (G-1) div (h-1)); dy = fl32((row (G-1) mod (h-1)) / (h-1)).
 *   grid_side  G, the side of the learned table (48), 1 .. 256
 *   idx4       device int32 [4, N] or NULL; w4 device float [4, N] or NULL;
 *   rowcol     device int32 [2, N] or NULL (row, col of each patch).
 * ------------------------------------------------------------------------- */
int ipe_vis_interp_plan(const int32_t *grid_thw_host, int n_images, int merge, int grid_side,
                        int32_t *idx4, float *w4, int32_t *rowcol, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_vis_pos_interp -- learned position table interpolated to each image's
 * patch grid, in merge order ([QVL] fast_pos_embed_interpolate; [CRT]
 * positions()):  out[k, :] = sum_c w_c(k) table[idx_c(k), :].
 * Frames of a video repeat frame 0.  Computed in fp32 as the separable form
 * (1-dx)((1-dy) T[y0,x0] + dy T[y1,x0]) + dx((1-dy) T[y0,x1] + dy T[y1,x1]),
 * equal to the four-weight sum in exact arithmetic, rounded once.
 *   table      device [G*G, hidden], dtype (row id = y G + x)
 *   hidden     channels, multiple of 4 (1152 in Qwen3-VL); at most
 *              65535 x 128 bytes (IPE_ELIMIT above)
 *   out        device [N, hidden], dtype, written; N = sum t h w.
 * ------------------------------------------------------------------------- */
int ipe_vis_pos_interp(const void *table, ipe_dtype dtype, int grid_side, int hidden,
                       const int32_t *grid_thw_host, int n_images, int merge, void *out,
                       void *stream);

/* ---------------------------------------------------------------------------
 * ipe_vis_pos_interp_hf -- ipe_vis_pos_interp with the rounding points of
 * the [QVL] fast_pos_embed_interpolate listing, run as written in the
 * table's dtype (same arguments):
 *   sample points torch.linspace(0, G-1, n) in fp32: step fl32((G-1)/(n-1)),
 *     point i = fl32(i step) for i < n/2, else fl32((G-1) - (n-1-i) step);
 *   y0 = trunc(y), y1 = min(y0 + 1, G-1), dy = y - y0 (fp32), likewise x;
 *   weights ((1-dy)(1-dx), (1-dy)dx, dy(1-dx), dy dx) as fp32 products, then
 *     rounded to the dtype;
 *   out = dtype(dtype(dtype(p0 + p1) + p2) + p3), p_c = dtype(T[idx_c] w_c),
 *     each sum taken in fp32 first.
 * hidden a multiple of 8 (bf16) or 4 (fp32); table and out 16-byte aligned
 * (IPE_EALIGN otherwise).
 * ------------------------------------------------------------------------- */
int ipe_vis_pos_interp_hf(const void *table, ipe_dtype dtype, int grid_side, int hidden,
                          const int32_t *grid_thw_host, int n_images, int merge, void *out,
                          void *stream);

/* ---------------------------------------------------------------------------
 * ipe_vis_rope2d -- vision 2-D rotary over the whole head, in place on q and k.
 * [QVL] rot_pos_emb + apply_rotary_pos_emb_vision; [CRT] rope_angles(),
 * attention():  with f = head_dim/4 frequencies inv[i] = fl32(1/theta^(2i/(head_dim/2)))
 * and (row, col) the patch's grid position, angle a[i] = fl32(row * inv[i]),
 * a[f + i] = fl32(col * inv[i]) (i < f), and for j < head_dim/2:
 *   x'[j] = x[j] cos a[j] - x[j + head_dim/2] sin a[j]
 *   x'[j + head_dim/2] = x[j + head_dim/2] cos a[j] + x[j] sin a[j].
 * One sincosf per (patch, angle), shared by every head of q and k.
 *   q, k       device [n_patch, heads, head_dim], dtype; heads contiguous;
 *              patch strides q_stride, k_stride (>= heads * head_dim); k may be
 *              NULL (q only)
 *   n_patch    must equal sum t h w of grid_thw
 *   head_dim   multiple of 4 (72 in Qwen3-VL); theta > 0 (1e4).
 * ------------------------------------------------------------------------- */
int ipe_vis_rope2d(void *q, void *k, ipe_dtype dtype, int64_t n_patch, int heads, int head_dim,
                   int64_t q_stride, int64_t k_stride, const int32_t *grid_thw_host,
                   int n_images, int merge, double theta, void *stream);

/* ---------------------------------------------------------------------------
 * ipe_vis_pos_interp_rope2d -- ipe_vis_pos_interp and ipe_vis_rope2d on the
 * same images in one call: the interpolation runs on a second stream of the
 * library (one per device, created on first use) while the rotation runs on
 * `stream`, so the two kernels share the SMs; `stream` waits for both.  The
 * rotation is launched first, with shared-memory blocks small enough to
 * leave room for two interpolation blocks on every SM where that still
 * gives it a two-stage ring.  Same results as the two calls.  Arguments as
 * for the two calls; one dtype for table, out, q and k.
 * ------------------------------------------------------------------------- */
int ipe_vis_pos_interp_rope2d(const void *table, int grid_side, int hidden, void *out, void *q,
                              void *k, int heads, int head_dim, int64_t q_stride, int64_t k_stride,
                              double theta, ipe_dtype dtype, const int32_t *grid_thw_host,
                              int n_images, int merge, void *stream);

/* ---------------------------------------------------------------------------
 * Host-buffer entry points.  Not part of any page: the streaming runtime of
 * this library around the same kernels.  The data moves host -> device,
 * through the kernel and back in chunks, so that both copy directions and
 * the kernels overlap:
 *   copies in   on a library copy stream (one per device),
 *   the kernel  on `stream`, after its chunk's copies in,
 *   copies out  on a second library copy stream, after the kernel.
 * Consecutive calls share the copy streams, so one call's copies also
 * overlap the next call's.  Results are exactly those of the device entry
 * points (the same kernels on each chunk).
 *   *_host      host buffers; page-locked memory gives the overlap
 *               (pageable memory works without it).  The out buffers may be
 *               the in buffers.
 *   *_dev       device staging buffers of the full size, caller-owned.  The
 *               library remembers, per staging buffer, where the last
 *               copies out of it end; a later call waits for them before
 *               copying in again.
 *   join        non-zero: `stream` waits for every copy out enqueued so far
 *               on the device, so its completion means the results are in
 *               host memory; zero: use ipe_host_join or a later call with
 *               join set.
 * The first call on a device creates its two copy streams and their events.
 * Argument checks of the device calls apply to every chunk; a failed chunk
 * stops the call with its status (earlier chunks stay enqueued).
 * ------------------------------------------------------------------------- */

/* `stream` waits for every copy out enqueued so far on the current device. */
int ipe_host_join(void *stream);

/* ipe_mrope_apply on host q [T, hq, head_dim] / k [T, hk, head_dim]
 * (contiguous) and host positions [3, T], chunk_tokens tokens at a time;
 * q_dev / k_dev: [T, hq / hk, head_dim]; positions_dev: 3 T int32 (each
 * chunk's positions stored as [3, n] at offset 3 t0). */
int ipe_mrope_apply_host(const void *q_host, const void *k_host, void *q_out_host, void *k_out_host,
                         ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                         const int32_t *positions_host, const float *inv_freq_host, int rot_dim,
                         const int32_t *section, int interleaved, void *q_dev, void *k_dev,
                         int32_t *positions_dev, int64_t chunk_tokens, int join, void *stream);

/* ipe_vis_rope2d on host q / k [N, heads, head_dim] (contiguous); chunks of
 * whole images up to chunk_rows patches, an image above that split into
 * frame ranges.  k_host / k_out_host / k_dev may be NULL together. */
int ipe_vis_rope2d_host(const void *q_host, const void *k_host, void *q_out_host, void *k_out_host,
                        ipe_dtype dtype, int heads, int head_dim, const int32_t *grid_thw_host,
                        int n_images, int merge, double theta, void *q_dev, void *k_dev,
                        int64_t chunk_rows, int join, void *stream);

/* ipe_vis_pos_interp from a host table [G*G, hidden] to host out [N, hidden];
 * the table moves in once, the output comes back in chunks as for
 * ipe_vis_rope2d_host. */
int ipe_vis_pos_interp_host(const void *table_host, ipe_dtype dtype, int grid_side, int hidden,
                            const int32_t *grid_thw_host, int n_images, int merge, void *out_host,
                            void *table_dev, void *out_dev, int64_t chunk_rows, int join, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* IPE_H */
