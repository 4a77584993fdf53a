/*
 * oracle.c -- plain, slow, double-precision CPU statement of the positional
 * encoding path of the Qwen3-VL / Qwen3.5 vision-language pipeline.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or execute this file; only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Every function follows the steps of the page it cites, in that page's
 * order and notation, with no blocking, fusion or reordering.  Arithmetic is
 * IEEE double, except where the pages fix an fp32 step (the fp32 outer
 * product of positions and inverse frequencies): that step is evaluated
 * exactly as fp32 would, by forming the product of two fp32 values in double
 * (exact: 24 + 24 significant bits fit in 53) and rounding it once to fp32.
 *
 * Pages cited (title -- section):
 *   [QVL]  "Qwen3-VL" notes, frankmowj.github.io -- fast_pos_embed_interpolate,
 *          apply_rotary_pos_emb_vision, Qwen3VLVisionModel.rot_pos_emb,
 *          Qwen3VLTextRotaryEmbedding (apply_interleaved_mrope, forward)
 *   [IRPE] "Interleaved Rotary Position Embedding", taking-lying-flat.github.io
 *          -- compute_default_rope_parameters, rotate_half /
 *          apply_rotary_pos_emb, recomposition_frequencies
 *   [M01]  "M01 RMSNorm and multimodal RoPE (interleaved / chunked)",
 *          kuanzhou.online nano-vllm-omni drills -- problem summary, shape
 *          trace, step-by-step axis figure, L1 hints
 *   [CRT]  cortiq-engine 0.8.52 src/qwen3vis.rs, docs.rs -- positions(),
 *          rope_angles(), attention()
 *
 * Parity status: every function here is pinned by the not-gpu tests (worked
 * values printed on the pages, closed forms, invariants, brute force).  The
 * vision 2-D rotary has no printed numeric example; it is pinned by
 * invariants, a basis-vector read-back, and the pages' rot_pos_emb /
 * apply_rotary_pos_emb_vision steps evaluated by torch in fp32.  The text
 * cos / sin are also pinned to both printed forms of the interleaved
 * selection ([QVL] apply_interleaved_mrope before the cos, [IRPE]
 * recomposition_frequencies after it) evaluated by torch in fp32.
 *
 * Return convention: 0 on success, -1 on an argument the definition does not
 * cover.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* fp32 rounding of a double (round to nearest even, the C default). */
static float f32(double v) { return (float)v; }

/* Exact fp32 product: both operands are fp32, their double product is exact,
 * one rounding to fp32 follows. */
static float f32_mul(float a, float b) { return (float)((double)a * (double)b); }

/* ------------------------------------------------------------------------
 * Default RoPE inverse frequencies.
 * [IRPE] compute_default_rope_parameters; [M01] problem summary:
 *   inv_freq = 1 / base ** (arange(0, dim, 2) / dim)
 * Reading: the power and the reciprocal are taken in double and the result is
 * rounded once to fp32 (the pages compute it in fp32 and keep it in fp32).
 * Writes one value per even k in [0, dim).  Returns the count written.
 * ---------------------------------------------------------------------- */
int orc_rope_inv_freq(int dim, double base, float *inv_freq)
{
    if (dim <= 0 || !(base > 0.0))
        return -1;
    int n = 0;
    for (int k = 0; k < dim; k += 2) {
        double exponent = (double)k / (double)dim;
        inv_freq[n++] = f32(1.0 / pow(base, exponent));
    }
    return n;
}

/* ------------------------------------------------------------------------
 * Per-frequency axis selection over a [3][rows][half] tensor of candidates.
 *
 * Interleaved, [QVL] apply_interleaved_mrope / [IRPE]
 * recomposition_frequencies: start from the T plane (a copy), then for
 * dim = 1 (H), 2 (W) with offset = dim, overwrite the columns of
 * slice(offset, 3 * mrope_section[dim], 3) with that axis' plane.  Python
 * slice semantics: the stop is clipped to the axis length.
 *
 * Chunked, [M01] step-by-step figure: concatenate the column ranges
 * [0, s_t) of T, [s_t, s_t + s_h) of H and [s_t + s_h, half) of W, the same
 * column range of each axis.
 *
 * Reading: mrope_section must sum to half ([M01] problem summary: "the sum
 * is D/2"); anything else is rejected.
 * ---------------------------------------------------------------------- */
static int select_axis_columns(const double *cand, int64_t rows, int half,
                               const int section[3], int interleaved, double *out)
{
    if (section[0] < 0 || section[1] < 0 || section[2] < 0)
        return -1;
    if (section[0] + section[1] + section[2] != half)
        return -1;
    const int64_t plane = rows * (int64_t)half;
    if (interleaved) {
        /* freqs_t = freqs[0] (copied so the source plane stays intact) */
        memcpy(out, cand, (size_t)plane * sizeof(double));
        for (int dim = 1; dim <= 2; ++dim) {
            int offset = dim;
            int length = section[dim] * 3;
            int stop = length < half ? length : half;
            for (int idx = offset; idx < stop; idx += 3)
                for (int64_t r = 0; r < rows; ++r)
                    out[r * half + idx] = cand[dim * plane + r * half + idx];
        }
    } else {
        int col = 0;
        for (int a = 0; a < 3; ++a) {
            for (int c = col; c < col + section[a]; ++c)
                for (int64_t r = 0; r < rows; ++r)
                    out[r * half + c] = cand[a * plane + r * half + c];
            col += section[a];
        }
    }
    return 0;
}

/* Axis label (0 = T, 1 = H, 2 = W) of every frequency: the selection above
 * applied to planes filled with their own axis number. */
int orc_mrope_axis_labels(int half, const int section[3], int interleaved, int *axis)
{
    if (half <= 0)
        return -1;
    double *cand = (double *)malloc(sizeof(double) * 3 * (size_t)half);
    double *sel = (double *)malloc(sizeof(double) * (size_t)half);
    for (int a = 0; a < 3; ++a)
        for (int j = 0; j < half; ++j)
            cand[a * half + j] = (double)a;
    int rc = select_axis_columns(cand, 1, half, section, interleaved, sel);
    if (rc == 0)
        for (int j = 0; j < half; ++j)
            axis[j] = (int)sel[j];
    free(cand);
    free(sel);
    return rc;
}

/* ------------------------------------------------------------------------
 * Multimodal RoPE cos / sin.
 * [QVL] Qwen3VLTextRotaryEmbedding.forward; [M01] shape trace rows 2-7:
 *   freqs[a, t, i] = float(positions[a, t]) * inv_freq[i]   (fp32, autocast off)
 *   f = axis selection of freqs                               -> [T, half]
 *   emb = cat(f, f, -1)                                       -> [T, 2 half]
 *   cos = emb.cos() * attention_scaling, sin = emb.sin() * attention_scaling
 * attention_scaling is 1 for the default rope type ([IRPE]
 * compute_default_rope_parameters).  cos / sin are taken in double of the
 * fp32 angle.
 * positions: [3][T] (rows t, h, w).  cos_out, sin_out: [T][2 half].
 * ---------------------------------------------------------------------- */
int orc_mrope_cos_sin(const int64_t *positions, int64_t T, const float *inv_freq, int half,
                      const int section[3], int interleaved, double *cos_out, double *sin_out)
{
    if (T < 0 || half <= 0)
        return -1;
    if (T == 0)
        return section[0] + section[1] + section[2] == half ? 0 : -1;
    const int64_t plane = T * (int64_t)half;
    double *freqs = (double *)malloc(sizeof(double) * 3 * (size_t)plane);
    double *f = (double *)malloc(sizeof(double) * (size_t)plane);
    for (int a = 0; a < 3; ++a)
        for (int64_t t = 0; t < T; ++t) {
            float p = f32((double)positions[a * T + t]);
            for (int i = 0; i < half; ++i)
                freqs[a * plane + t * half + i] = (double)f32_mul(p, inv_freq[i]);
        }
    int rc = select_axis_columns(freqs, T, half, section, interleaved, f);
    if (rc == 0) {
        const double attention_scaling = 1.0;
        for (int64_t t = 0; t < T; ++t)
            for (int j = 0; j < 2 * half; ++j) {
                double emb = f[t * half + (j < half ? j : j - half)];
                cos_out[t * 2 * half + j] = cos(emb) * attention_scaling;
                sin_out[t * 2 * half + j] = sin(emb) * attention_scaling;
            }
    }
    free(freqs);
    free(f);
    return rc;
}

/* ------------------------------------------------------------------------
 * rotate_half and partial apply_rotary_pos_emb.
 * [IRPE] rotate_half / apply_rotary_pos_emb; [M01] L1 hints:
 *   rotate_half(x) = cat(-x[..., d/2:], x[..., :d/2])
 *   x_rot, x_pass = x[..., :rot], x[..., rot:]   with rot = cos.shape[-1]
 *   out = cat(x_rot * cos + rotate_half(x_rot) * sin, x_pass)
 * cos / sin are [T][rot] and broadcast over the heads (unsqueeze on the head
 * axis).  x, out: [T][H][D].  mag (optional): [T][H][rot], the sum of the
 * magnitudes of the two products of each output, |x_rot cos| + |rh sin|,
 * for the error model of the tests.
 * ---------------------------------------------------------------------- */
void orc_rotate_half(const double *x, int d, double *out)
{
    int h = d / 2;
    for (int j = 0; j < d; ++j)
        out[j] = j < h ? -x[j + h] : x[j - h];
}

int orc_apply_rotary(const double *x, int64_t T, int H, int D, const double *cos_v,
                     const double *sin_v, int rot, double *out, double *mag)
{
    if (T < 0 || H < 0 || D <= 0 || rot < 0 || rot > D || (rot & 1))
        return -1;
    double *rh = (double *)malloc(sizeof(double) * (size_t)(rot > 0 ? rot : 1));
    for (int64_t t = 0; t < T; ++t)
        for (int hd = 0; hd < H; ++hd) {
            const double *xr = x + (t * H + hd) * (int64_t)D;
            double *o = out + (t * H + hd) * (int64_t)D;
            orc_rotate_half(xr, rot, rh);
            for (int j = 0; j < rot; ++j) {
                double a = xr[j] * cos_v[t * rot + j];
                double b = rh[j] * sin_v[t * rot + j];
                o[j] = a + b;
                if (mag)
                    mag[(t * H + hd) * (int64_t)rot + j] = fabs(a) + fabs(b);
            }
            for (int j = rot; j < D; ++j)
                o[j] = xr[j];
        }
    free(rh);
    return 0;
}

/* ------------------------------------------------------------------------
 * Vision position-table interpolation.
 * [QVL] fast_pos_embed_interpolate, with [CRT] positions() for n = 1:
 *   h_idxs = linspace(0, G - 1, h), w_idxs likewise      (G = num_grid_per_side)
 *   floor = int(idx), ceil = clip(floor + 1, max = G - 1), d = idx - floor
 *   corners (TL, TR, BL, BR) = (fh G + fw, fh G + cw, ch G + fw, ch G + cw)
 *   weights = ((1-dh)(1-dw), (1-dh) dw, dh (1-dw), dh dw)
 *   patch_pos_embeds = sum_k pos_embed[idx_k] * weight_k      -> [h w, C]
 *   per image: repeat(t, 1), view(t, h/m, m, w/m, m, C),
 *              permute(0, 1, 3, 2, 4, 5), flatten; images concatenated.
 * Reading: the sample coordinate is the exact rational i (G-1)/(n-1)
 * (0 when n = 1) in double instead of fp32 linspace; weights and sums are
 * double.
 * ---------------------------------------------------------------------- */
static double linspace_at(int G, int n, int i)
{
    if (n == 1)
        return 0.0;
    return (double)i * (double)(G - 1) / (double)(n - 1);
}

static int check_grid(const int *grid_thw, int n_images, int m, int64_t *total)
{
    if (n_images < 0 || m <= 0)
        return -1;
    int64_t N = 0;
    for (int i = 0; i < n_images; ++i) {
        int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        if (t <= 0 || h <= 0 || w <= 0 || h % m || w % m)
            return -1;
        N += (int64_t)t * h * w;
    }
    *total = N;
    return 0;
}

int64_t orc_grid_patches(const int *grid_thw, int n_images, int m)
{
    int64_t N;
    return check_grid(grid_thw, n_images, m, &N) ? -1 : N;
}

/* Corner ids and weights of one image in raster order: idx[4][h w], wt[4][h w]. */
static void bilinear_corners(int G, int h, int w, int64_t *idx, double *wt)
{
    int64_t hw = (int64_t)h * w;
    for (int y = 0; y < h; ++y) {
        double hy = linspace_at(G, h, y);
        int h_floor = (int)hy;
        int h_ceil = h_floor + 1 > G - 1 ? G - 1 : h_floor + 1;
        double dh = hy - h_floor;
        int64_t base_h = (int64_t)h_floor * G, base_h_ceil = (int64_t)h_ceil * G;
        for (int x = 0; x < w; ++x) {
            double wx = linspace_at(G, w, x);
            int w_floor = (int)wx;
            int w_ceil = w_floor + 1 > G - 1 ? G - 1 : w_floor + 1;
            double dw = wx - w_floor;
            int64_t k = (int64_t)y * w + x;
            idx[0 * hw + k] = base_h + w_floor;
            idx[1 * hw + k] = base_h + w_ceil;
            idx[2 * hw + k] = base_h_ceil + w_floor;
            idx[3 * hw + k] = base_h_ceil + w_ceil;
            wt[0 * hw + k] = (1 - dh) * (1 - dw);
            wt[1 * hw + k] = (1 - dh) * dw;
            wt[2 * hw + k] = dh * (1 - dw);
            wt[3 * hw + k] = dh * dw;
        }
    }
}

/* Row of the t-repeated raster buffer that lands at each output row of one
 * image after view(t, h/m, m, w/m, m).permute(0, 1, 3, 2, 4, 5).flatten():
 * the loops run over the permuted axes (t, h/m, w/m, m, m) and the source
 * index is the view's own linear index of (a, b, c, d, e). */
static void merge_permute_rows(int t, int h, int w, int m, int64_t *src_row)
{
    int64_t k = 0;
    int hb = h / m, wb = w / m;
    for (int a = 0; a < t; ++a)
        for (int b = 0; b < hb; ++b)
            for (int d = 0; d < wb; ++d)
                for (int c = 0; c < m; ++c)
                    for (int e = 0; e < m; ++e) {
                        int64_t view_index = ((((int64_t)a * hb + b) * m + c) * wb + d) * m + e;
                        src_row[k++] = view_index;
                    }
}

int orc_vis_pos_embed_interpolate(const double *pos_embed, int G, int C, const int *grid_thw,
                                  int n_images, int m, double *out, double *mag)
{
    int64_t N;
    if (G <= 0 || C <= 0 || check_grid(grid_thw, n_images, m, &N))
        return -1;
    int64_t row0 = 0;
    for (int i = 0; i < n_images; ++i) {
        int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        int64_t hw = (int64_t)h * w;
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * 4 * (size_t)hw);
        double *wt = (double *)malloc(sizeof(double) * 4 * (size_t)hw);
        double *flat = (double *)malloc(sizeof(double) * (size_t)(hw * C));
        double *flat_mag = (double *)malloc(sizeof(double) * (size_t)(hw * C));
        bilinear_corners(G, h, w, idx, wt);
        for (int64_t k = 0; k < hw; ++k)
            for (int c = 0; c < C; ++c) {
                double s = 0.0, sa = 0.0;
                for (int q = 0; q < 4; ++q) {
                    double term = pos_embed[idx[q * hw + k] * C + c] * wt[q * hw + k];
                    s += term;
                    sa += fabs(term);
                }
                flat[k * C + c] = s;
                flat_mag[k * C + c] = sa;
            }
        /* repeat(t, 1): repeated row r is raster row r mod (h w) */
        int64_t *src = (int64_t *)malloc(sizeof(int64_t) * (size_t)(t * hw));
        merge_permute_rows(t, h, w, m, src);
        for (int64_t k = 0; k < t * hw; ++k) {
            int64_t r = src[k] % hw;
            memcpy(out + (row0 + k) * C, flat + r * C, sizeof(double) * (size_t)C);
            if (mag)
                memcpy(mag + (row0 + k) * C, flat_mag + r * C, sizeof(double) * (size_t)C);
        }
        row0 += t * hw;
        free(idx);
        free(wt);
        free(flat);
        free(flat_mag);
        free(src);
    }
    return 0;
}

/* Corner ids [4][N] and weights [4][N] in output (merge) order, for the
 * bit-exact index check.  Same steps as above, applied to the index and
 * weight lists instead of the table rows. */
int orc_vis_interp_plan(const int *grid_thw, int n_images, int m, int G, int64_t *idx4, double *w4)
{
    int64_t N;
    if (G <= 0 || check_grid(grid_thw, n_images, m, &N))
        return -1;
    int64_t row0 = 0;
    for (int i = 0; i < n_images; ++i) {
        int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        int64_t hw = (int64_t)h * w;
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * 4 * (size_t)hw);
        double *wt = (double *)malloc(sizeof(double) * 4 * (size_t)hw);
        int64_t *src = (int64_t *)malloc(sizeof(int64_t) * (size_t)(t * hw));
        bilinear_corners(G, h, w, idx, wt);
        merge_permute_rows(t, h, w, m, src);
        for (int64_t k = 0; k < t * hw; ++k) {
            int64_t r = src[k] % hw;
            for (int q = 0; q < 4; ++q) {
                idx4[q * N + row0 + k] = idx[q * hw + r];
                w4[q * N + row0 + k] = wt[q * hw + r];
            }
        }
        row0 += t * hw;
        free(idx);
        free(wt);
        free(src);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Vision (row, col) per patch.
 * [QVL] Qwen3VLVisionModel.rot_pos_emb:
 *   row_idx = block_rows[:, None, None, None] * m + intra_row[None, None, :, None]
 *   col_idx = block_cols[None, :, None, None] * m + intra_col[None, None, None, :]
 *   both expanded to (merged_h, merged_w, m, m) and flattened; stacked to
 *   (row, col); repeated num_frames times; images concatenated.
 * pos_ids: [N][2].
 * ---------------------------------------------------------------------- */
int orc_vis_rot_pos_ids(const int *grid_thw, int n_images, int m, int64_t *pos_ids)
{
    int64_t N;
    if (check_grid(grid_thw, n_images, m, &N))
        return -1;
    int64_t off = 0;
    for (int i = 0; i < n_images; ++i) {
        int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        int merged_h = h / m, merged_w = w / m;
        int64_t n_tok = (int64_t)merged_h * merged_w * m * m;
        int64_t k = 0;
        for (int br = 0; br < merged_h; ++br)
            for (int bc = 0; bc < merged_w; ++bc)
                for (int ir = 0; ir < m; ++ir)
                    for (int ic = 0; ic < m; ++ic) {
                        pos_ids[2 * (off + k)] = (int64_t)br * m + ir;
                        pos_ids[2 * (off + k) + 1] = (int64_t)bc * m + ic;
                        ++k;
                    }
        for (int f = 1; f < t; ++f)
            memcpy(pos_ids + 2 * (off + f * n_tok), pos_ids + 2 * off, sizeof(int64_t) * 2 * (size_t)n_tok);
        off += t * n_tok;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Vision rotary cos / sin.
 * [QVL] rot_pos_emb: freq_table = rotary_pos_emb(max_hw) is the fp32 outer
 * product of arange(max_hw) and the 18 inverse frequencies of dim
 * head_dim / 2 (= 36); embeddings = freq_table[pos_ids].flatten(1) -> [N, 36]
 * (18 row angles then 18 column angles, as [CRT] rope_angles() spells out).
 * [QVL] apply_rotary_pos_emb_vision uses emb = cat(embeddings, embeddings)
 * -> [N, head_dim] and its cos / sin.  theta is the vision rope base (1e4).
 * Reading: angles are fl32(fl32(index) * inv_freq_f32), the same rule as the
 * text path; cos / sin in double.
 * cos_out, sin_out: [N][head_dim].
 * ---------------------------------------------------------------------- */
int orc_vis_rotary_cos_sin(const int64_t *pos_ids, int64_t N, int head_dim, double theta,
                           double *cos_out, double *sin_out)
{
    if (N < 0 || head_dim <= 0 || head_dim % 4)
        return -1;
    int dim = head_dim / 2;     /* 36 */
    int nf = dim / 2;           /* 18 per axis */
    float *inv = (float *)malloc(sizeof(float) * (size_t)nf);
    orc_rope_inv_freq(dim, theta, inv);
    for (int64_t p = 0; p < N; ++p)
        for (int j = 0; j < head_dim; ++j) {
            int e = j < dim ? j : j - dim;   /* cat(emb, emb) */
            int axis = e < nf ? 0 : 1;       /* flatten of [2, 18] */
            int i = e < nf ? e : e - nf;
            float angle = f32_mul(f32((double)pos_ids[2 * p + axis]), inv[i]);
            cos_out[p * head_dim + j] = cos((double)angle);
            sin_out[p * head_dim + j] = sin((double)angle);
        }
    free(inv);
    return 0;
}

/* ------------------------------------------------------------------------
 * RMSNorm over the last axis, in the order the drill page fixes.
 * [M01] problem summary and L2 hints (rms_norm):
 *   x32 = float(x); xn = x32 * rsqrt(mean(x32^2, -1, keepdim) + eps)
 *   y = xn.to(x.dtype) * weight            (cast back first, then the weight)
 * Reading: mean, rsqrt and the product are taken in double; the two casts are
 * the dtype's own rounding (dtype 0: fp32, 1: bf16, round to nearest even),
 * the second applied to the exact product of the two rounded values.
 * x, out: [R][D]; weight: [D] (values of the weight's dtype).
 * ---------------------------------------------------------------------- */
static double round_to(double v, int dtype)
{
    if (dtype == 0)
        return (double)(float)v;
    /* bf16: round the fp32-representable value v to 8 significant bits, ties
     * to even, through its fp32 bit pattern (v is first rounded to fp32, as
     * the dtype conversion of a fp32 tensor does) */
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u)
        return (double)f;
    uint32_t r = u + 0x7fffu + ((u >> 16) & 1u);
    r &= 0xffff0000u;
    float g;
    memcpy(&g, &r, sizeof g);
    return (double)g;
}

int orc_rms_norm(const double *x, int64_t R, int D, const double *weight, double eps, int dtype, double *out)
{
    if (R < 0 || D <= 0 || (dtype != 0 && dtype != 1) || eps < 0)
        return -1;
    for (int64_t r = 0; r < R; ++r) {
        const double *xr = x + r * D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d)
            ss += xr[d] * xr[d];
        double inv = 1.0 / sqrt(ss / D + eps);
        for (int d = 0; d < D; ++d) {
            double xn = round_to(xr[d] * inv, dtype);            /* .to(x.dtype) */
            out[r * D + d] = round_to(xn * weight[d], dtype);    /* * weight */
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Three-axis position table of a batch of mixed sequences, and the per-sample
 * rope deltas.
 * [IRPE] get_rope_index(): preparing the grids, filtering padding and
 * splitting runs, advancing the position, flattening the vision grid,
 * joining the sequence back, returning positions and deltas; and the worked
 * single-batch table.  [IRPE] mm_tokens gives the type codes: 0 text (and
 * message / media start-end markers), 1 image, 2 video, 3 audio.
 *
 * Steps, in the page's order:
 *  1. every video grid row (t, h, w) becomes t rows (1, h, w), one per
 *     temporal slice; image rows are used as they are;
 *  2. one image iterator and one video iterator serve the whole batch, in
 *     the order of samples and of appearance within a sample;
 *  3. per sample: keep the slots whose mask is non-zero, split the kept
 *     type sequence into runs of equal consecutive type;
 *  4. current_pos starts at 0; a text run of n slots gets arange(n) +
 *     current_pos on all three rows and advances current_pos by n; a vision
 *     run takes the next grid of its kind, lays out llm_t = t, llm_h = h / m,
 *     llm_w = w / m slots width-fastest with coordinates
 *     (current_pos + tt, current_pos + row, current_pos + col) and advances
 *     current_pos by max(h, w) / m (not by its slot count);
 *  5. the runs are joined and written back to the kept slots; padded slots
 *     stay 0; the delta is max(joined) + 1 - (number of kept slots).
 * Readings: an audio run (type 3) is laid out like text -- the page on the
 * Omni drills states that audio positions advance linearly in time, and the
 * listing has no grid for it.  A sample with no kept slot gets delta 0 (the
 * listing would take the maximum of an empty table).
 *
 * types, mask: [B][L] (mask may be NULL: every slot kept); img_grid: [n_img][3];
 * vid_grid: [n_vid][3]; pos: [3][B][L]; deltas: [B].
 * Returns 0; -1 on bad arguments; -2 when a vision run finds its iterator
 * exhausted; -3 when the joined table of a sample does not have one column
 * per kept slot.
 * ---------------------------------------------------------------------- */
int orc_rope_index(const int64_t *types, const int64_t *mask, int B, int64_t L, const int64_t *img_grid,
                   int n_img, const int64_t *vid_grid, int n_vid, int m, int64_t *pos, int64_t *deltas)
{
    if (B < 0 || L < 0 || n_img < 0 || n_vid < 0 || m <= 0)
        return -1;
    /* 1. video grids repeated per temporal slice, t set to 1 */
    int64_t n_slices = 0;
    for (int v = 0; v < n_vid; ++v) {
        if (vid_grid[3 * v] < 0)
            return -1;
        n_slices += vid_grid[3 * v];
    }
    int64_t *slices = malloc(sizeof(int64_t) * 3 * (size_t)(n_slices > 0 ? n_slices : 1));
    int64_t *kept = malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
    int64_t *table = malloc(sizeof(int64_t) * 3 * (size_t)(L > 0 ? L : 1));
    if (!slices || !kept || !table) {
        free(slices);
        free(kept);
        free(table);
        return -1;
    }
    int64_t s = 0;
    for (int v = 0; v < n_vid; ++v)
        for (int64_t r = 0; r < vid_grid[3 * v]; ++r, ++s) {
            slices[3 * s] = 1;
            slices[3 * s + 1] = vid_grid[3 * v + 1];
            slices[3 * s + 2] = vid_grid[3 * v + 2];
        }
    for (int64_t i = 0; i < 3 * (int64_t)B * L; ++i)
        pos[i] = 0;
    /* 2. iterators shared by the batch */
    int64_t next_img = 0, next_vid = 0;
    int rc = 0;
    for (int b = 0; b < B && rc == 0; ++b) {
        /* 3. kept slots (their indices into the padded row) */
        int64_t n = 0;
        for (int64_t l = 0; l < L; ++l)
            if (mask == NULL || mask[(int64_t)b * L + l] != 0)
                kept[n++] = l;
        /* 4. runs of equal type over the kept sequence, current_pos from 0 */
        int64_t cur = 0, cols = 0;
        int64_t start = 0;
        while (start < n && rc == 0) {
            int64_t key = types[(int64_t)b * L + kept[start]];
            int64_t end = start + 1;
            while (end < n && types[(int64_t)b * L + kept[end]] == key)
                ++end;
            if (key == 0 || key == 3) {
                int64_t text_len = end - start;
                for (int64_t i = 0; i < text_len; ++i) {
                    if (cols >= n) {
                        rc = -3;
                        break;
                    }
                    for (int a = 0; a < 3; ++a)
                        table[a * n + cols] = i + cur;
                    ++cols;
                }
                cur += text_len;
            } else if (key == 1 || key == 2) {
                const int64_t *g;
                if (key == 1) {
                    if (next_img >= n_img) {
                        rc = -2;
                        break;
                    }
                    g = img_grid + 3 * next_img++;
                } else {
                    if (next_vid >= n_slices) {
                        rc = -2;
                        break;
                    }
                    g = slices + 3 * next_vid++;
                }
                int64_t lt = g[0], lh = g[1] / m, lw = g[2] / m;
                for (int64_t tt = 0; tt < lt; ++tt)
                    for (int64_t hh = 0; hh < lh; ++hh)
                        for (int64_t ww = 0; ww < lw; ++ww) {
                            if (cols >= n) {
                                rc = -3;
                                break;
                            }
                            table[0 * n + cols] = tt * 1 + cur;   /* time_interval 1 */
                            table[1 * n + cols] = hh + cur;
                            table[2 * n + cols] = ww + cur;
                            ++cols;
                        }
                cur += (g[1] > g[2] ? g[1] : g[2]) / m;
            } else {
                rc = -1;
            }
            start = end;
        }
        if (rc == 0 && cols != n)
            rc = -3;
        if (rc != 0)
            break;
        /* 5. write back to kept slots; delta from the joined table */
        int64_t mx = 0;
        for (int64_t c = 0; c < n; ++c)
            for (int a = 0; a < 3; ++a) {
                pos[((int64_t)a * B + b) * L + kept[c]] = table[a * n + c];
                if ((c == 0 && a == 0) || table[a * n + c] > mx)
                    mx = table[a * n + c];
            }
        deltas[b] = n > 0 ? mx + 1 - n : 0;
    }
    free(slices);
    free(kept);
    free(table);
    return rc;
}

/* ------------------------------------------------------------------------
 * Positions of the tokens of a generation step, from the sequence index and
 * the rope deltas saved at prefill.
 * [IRPE] compute_3d_position_ids(), "recovering the positions": with a
 * padding mask the sequence index is cumsum(mask, -1) - 1 with the padded
 * slots set to 0; without one it is arange from the cache length.  The index
 * is expanded to three rows and the sample's delta is added; all three axes
 * then carry the same text position.
 * mask: [B][S] over the whole sequence so far, the n_new new tokens last (or
 * NULL: cache_len[b] + i); deltas: [B] (or NULL: 0); pos: [3][B][n_new].
 * ---------------------------------------------------------------------- */
int orc_decode_positions(const int64_t *mask, int B, int64_t S, const int64_t *cache_len, int64_t n_new,
                         const int64_t *deltas, int64_t *pos)
{
    if (B < 0 || n_new < 0 || (mask != NULL && (S < n_new)) || (mask == NULL && cache_len == NULL))
        return -1;
    for (int b = 0; b < B; ++b) {
        int64_t run = 0;   /* cumsum of the mask up to the current slot */
        for (int64_t i = 0; i < (mask ? S : n_new); ++i) {
            int64_t seq;
            if (mask) {
                run += mask[(int64_t)b * S + i];
                seq = mask[(int64_t)b * S + i] == 0 ? 0 : run - 1;
                if (i < S - n_new)
                    continue;
            } else {
                seq = cache_len[b] + i;
            }
            int64_t col = mask ? i - (S - n_new) : i;
            for (int a = 0; a < 3; ++a)
                pos[((int64_t)a * B + b) * n_new + col] = seq + (deltas ? deltas[b] : 0);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * HF rounding mode (the rounding points of the listings run as written in
 * the activation dtype), for users who must match those checkpoints bit
 * for bit.
 *
 * Interpolation.  [QVL] fast_pos_embed_interpolate: the sample coordinates
 * are an fp32 linspace (passed in: ys[h], xs[w] per image, concatenated);
 * floor by truncation, ceiling min(floor + 1, G - 1); dh = y - floor in fp32;
 * the four weights (1-dh)(1-dw), (1-dh)dw, dh(1-dw), dh dw are fp32 products
 * and are then stored in the table's dtype; each corner row times its weight
 * is one dtype product, and the four products are summed left to right, each
 * sum rounded to the dtype (the dtype's arithmetic evaluates in fp32 and
 * rounds back); frames repeat, then the 6-D merge permute.
 * table: [G*G][C] values of the dtype; dtype 0 fp32, 1 bf16; out: [N][C].
 * ---------------------------------------------------------------------- */
int orc_vis_pos_interp_hf(const double *table, int G, int C, const int *grid_thw, int n_images, int m,
                          const float *ys, const float *xs, int dtype, double *out)
{
    int64_t total;
    if (G < 1 || C < 1 || (dtype != 0 && dtype != 1) || check_grid(grid_thw, n_images, m, &total))
        return -1;
    int64_t row0 = 0, yoff = 0, xoff = 0;
    for (int i = 0; i < n_images; ++i) {
        const int t = grid_thw[3 * i], h = grid_thw[3 * i + 1], w = grid_thw[3 * i + 2];
        const int64_t hw = (int64_t)h * w;
        double *frame = malloc(sizeof(double) * (size_t)(hw > 0 ? hw : 1) * C);
        int64_t *src = malloc(sizeof(int64_t) * (size_t)(hw > 0 ? hw : 1) * t);
        if (!frame || !src) {
            free(frame);
            free(src);
            return -1;
        }
        for (int r = 0; r < h; ++r)
            for (int c = 0; c < w; ++c) {
                const float y = ys[yoff + r], x = xs[xoff + c];
                const int y0 = (int)y, x0 = (int)x;               /* .int(): truncation */
                const int y1 = y0 + 1 < G - 1 ? y0 + 1 : G - 1;   /* .clip(max=G-1) */
                const int x1 = x0 + 1 < G - 1 ? x0 + 1 : G - 1;
                const float dh = y - (float)y0, dw = x - (float)x0;
                const float one_h = 1.0f - dh, one_w = 1.0f - dw;
                float wt[4] = {one_h * one_w, one_h * dw, dh * one_w, dh * dw};
                const int64_t idx[4] = {(int64_t)y0 * G + x0, (int64_t)y0 * G + x1, (int64_t)y1 * G + x0,
                                        (int64_t)y1 * G + x1};
                for (int q = 0; q < 4; ++q)
                    wt[q] = (float)round_to(wt[q], dtype);       /* weights in the table dtype */
                for (int ch = 0; ch < C; ++ch) {
                    double s = 0.0;
                    for (int q = 0; q < 4; ++q) {
                        const double p = round_to(table[idx[q] * C + ch] * (double)wt[q], dtype);
                        s = q == 0 ? p : round_to((double)((float)s + (float)p), dtype);
                    }
                    frame[((int64_t)r * w + c) * C + ch] = s;
                }
            }
        /* frames repeat frame 0, then the merge permute */
        merge_permute_rows(t, h, w, m, src);
        for (int64_t k = 0; k < (int64_t)t * hw; ++k)
            memcpy(out + (row0 + k) * C, frame + (src[k] % hw) * C, sizeof(double) * C);
        free(frame);
        free(src);
        row0 += (int64_t)t * hw;
        yoff += h;
        xoff += w;
    }
    (void)total;
    return 0;
}

/* Rotation.  [QVL] Qwen3VLTextRotaryEmbedding.forward returns cos and sin
 * cast to the activation dtype; [IRPE] apply_rotary_pos_emb computes
 * (q_rot * cos) + (rotate_half(q_rot) * sin) in that dtype; [M01] hints: for
 * bf16 inputs cos / sin are cast first, then multiplied.  Each product and
 * the sum are rounded to the dtype (the sum evaluated in fp32 first).
 * x: [T][H][D] values of the dtype; cos_v, sin_v: [T][rot] fp32 values. */
int orc_apply_rotary_hf(const double *x, int64_t T, int H, int D, const float *cos_v, const float *sin_v, int rot,
                        int dtype, double *out)
{
    if (T < 0 || H < 0 || rot < 2 || rot % 2 || rot > D || (dtype != 0 && dtype != 1))
        return -1;
    const int h = rot / 2;
    for (int64_t t = 0; t < T; ++t)
        for (int hd = 0; hd < H; ++hd) {
            const double *xr = x + (t * H + hd) * D;
            double *o = out + (t * H + hd) * D;
            for (int j = 0; j < rot; ++j) {
                const double c = round_to(cos_v[t * rot + j], dtype);
                const double s = round_to(sin_v[t * rot + j], dtype);
                const double rh = j < h ? -xr[j + h] : xr[j - h];      /* rotate_half */
                const double a = round_to(xr[j] * c, dtype);
                const double b = round_to(rh * s, dtype);
                o[j] = round_to((double)((float)a + (float)b), dtype);
            }
            memcpy(o + rot, xr + rot, sizeof(double) * (size_t)(D - rot));    /* pass-through */
        }
    return 0;
}
