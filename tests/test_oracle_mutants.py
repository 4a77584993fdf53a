"""Each plausible mistake planted in a copy of the oracle fails at least one pin.

The copy is compiled on the CPU into a temporary library; the committed
oracle is untouched.  A mutant whose original text is missing fails the test,
so the list stays in step with ``oracle/oracle.c``.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as obuild

import pins

MUTANTS = {
    # rotate_half written as [x2, -x1]: rotation in the wrong direction
    "rotate_half_sign": ("out[j] = j < h ? -x[j + h] : x[j - h];",
                         "out[j] = j < h ? x[j + h] : -x[j - h];"),
    # interleaved slice stop written as section instead of 3 * section
    "slice_stop": ("int length = section[dim] * 3;", "int length = section[dim];"),
    # H and W offsets exchanged
    "slice_offset": ("int offset = dim;", "int offset = 3 - dim;"),
    # chunked: H / W taken from column 0 of their plane instead of the same range
    "chunked_columns": ("out[r * half + c] = cand[a * plane + r * half + c];",
                        "out[r * half + c] = cand[a * plane + r * half + (c - col)];"),
    # every axis reads the T row of positions
    "positions_row": ("float p = f32((double)positions[a * T + t]);",
                      "float p = f32((double)positions[t]);"),
    # GPT-J style repeat_interleave instead of cat(f, f)
    "cat_vs_interleave": ("double emb = f[t * half + (j < half ? j : j - half)];",
                          "double emb = f[t * half + j / 2];"),
    # exponent arange(0, dim, 2) / dim written as arange(dim / 2) / dim
    "inv_freq_exponent": ("double exponent = (double)k / (double)dim;",
                          "double exponent = (double)(k / 2) / (double)dim;"),
    # pass-through channels dropped
    "pass_through": ("            o[j] = xr[j];\n", "            o[j] = 0.0;\n"),
    # linspace step (G-1)/n instead of (G-1)/(n-1)
    "linspace_step": ("return (double)i * (double)(G - 1) / (double)(n - 1);",
                      "return (double)i * (double)(G - 1) / (double)n;"),
    # top-right weight given the bottom-left formula
    "weight_swap": ("wt[1 * hw + k] = (1 - dh) * dw;", "wt[1 * hw + k] = dh * (1 - dw);"),
    # corner row base from the ceiling row for the top corners
    "corner_row": ("idx[1 * hw + k] = base_h + w_ceil;", "idx[1 * hw + k] = base_h_ceil + w_ceil;"),
    # merge permute (0,1,3,2,4,5) dropped: raster order
    "merge_permute": ("int64_t view_index = ((((int64_t)a * hb + b) * m + c) * wb + d) * m + e;",
                      "int64_t view_index = ((((int64_t)a * hb + b) * wb + d) * m + c) * m + e;"),
    # vision row index built from the intra-block column offset
    "rot_pos_row": ("pos_ids[2 * (off + k)] = (int64_t)br * m + ir;",
                    "pos_ids[2 * (off + k)] = (int64_t)br * m + ic;"),
    # vision angles: column angles first
    "vision_axis_order": ("int axis = e < nf ? 0 : 1;", "int axis = e < nf ? 1 : 0;"),
    # vision exponent 2i / head_dim instead of 2i / (head_dim / 2): the same
    # 18 values as base sqrt(theta) over dim (written so, to stay in bounds)
    "vision_inv_dim": ("orc_rope_inv_freq(dim, theta, inv);", "orc_rope_inv_freq(dim, sqrt(theta), inv);"),
    # RMSNorm: eps added after the square root
    "rms_eps_outside": ("double inv = 1.0 / sqrt(ss / D + eps);", "double inv = 1.0 / (sqrt(ss / D) + eps);"),
    # RMSNorm: the weight applied before the cast back to the dtype
    "rms_weight_before_cast": ("double xn = round_to(xr[d] * inv, dtype);", "double xn = xr[d] * inv;"),
    # RMSNorm: sum of squares instead of the mean
    "rms_sum_not_mean": ("double inv = 1.0 / sqrt(ss / D + eps);", "double inv = 1.0 / sqrt(ss + eps);"),
    # position table: a vision run advances by its slot count instead of its longer side
    "rope_advance_slots": ("cur += (g[1] > g[2] ? g[1] : g[2]) / m;", "cur += lt * lh * lw;"),
    # position table: padding kept (the mask ignored)
    "rope_mask_ignored": ("if (mask == NULL || mask[(int64_t)b * L + l] != 0)", "if (1)"),
    # position table: video grids not split into temporal slices
    "rope_video_slices": ("slices[3 * s] = 1;", "slices[3 * s] = vid_grid[3 * v];"),
    # position table: one image iterator per sample instead of per batch
    "rope_iter_per_sample": ("int64_t cur = 0, cols = 0;", "int64_t cur = 0, cols = 0;\n        next_img = 0;"),
    # position table: height and width coordinates exchanged
    "rope_hw_swap": ("table[1 * n + cols] = hh + cur;", "table[1 * n + cols] = ww + cur;"),
    # position table: delta taken against the padded length
    "rope_delta_padded": ("deltas[b] = n > 0 ? mx + 1 - n : 0;", "deltas[b] = n > 0 ? mx + 1 - L : 0;"),
    # decode positions: cumsum taken as the index (no - 1)
    "decode_cumsum": ("seq = mask[(int64_t)b * S + i] == 0 ? 0 : run - 1;",
                      "seq = mask[(int64_t)b * S + i] == 0 ? 0 : run;"),
    # decode positions: the rope delta not added
    "decode_no_delta": ("= seq + (deltas ? deltas[b] : 0);", "= seq;"),
    # HF interpolation: top-right and bottom-left weights exchanged
    "hf_weight_swap": ("float wt[4] = {one_h * one_w, one_h * dw, dh * one_w, dh * dw};",
                       "float wt[4] = {one_h * one_w, dh * one_w, one_h * dw, dh * dw};"),
    # HF interpolation: the running sum kept in double
    "hf_sum_unrounded": ("s = q == 0 ? p : round_to((double)((float)s + (float)p), dtype);",
                         "s = q == 0 ? p : s + p;"),
    # HF rotation: cos not cast to the activation dtype
    "hf_cos_unrounded": ("const double c = round_to(cos_v[t * rot + j], dtype);",
                         "const double c = cos_v[t * rot + j];"),
    # HF rotation: the product x cos not rounded
    "hf_product_unrounded": ("const double a = round_to(xr[j] * c, dtype);", "const double a = xr[j] * c;"),
    # position table: image temporal index dropped
    "angle_product_double": ("freqs[a * plane + t * half + i] = (double)f32_mul(p, inv_freq[i]);",
                             "freqs[a * plane + t * half + i] = (double)p * (double)inv_freq[i];"),
    "rope_image_time": ("table[0 * n + cols] = tt * 1 + cur;", "table[0 * n + cols] = cur;"),
}


def _failures(o):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except Exception:  # noqa: BLE001 - any error counts as a caught mutant
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")
    text = open(src).read()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutant {name}: original text not found exactly once"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(text.replace(old, new))
    lib = obuild.build(str(mutated), str(tmp_path / "liboracle_mutant.so"), force=True)
    failed = _failures(oracle.Oracle(lib))
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(tmp_path):
    src = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")
    shutil.copy(src, tmp_path / "oracle_copy.c")
    lib = obuild.build(str(tmp_path / "oracle_copy.c"), str(tmp_path / "liboracle_copy.so"), force=True)
    assert _failures(oracle.Oracle(lib)) == []
