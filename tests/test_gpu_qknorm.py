"""Fused QK-RMSNorm + MRoPE (through the C ABI) against the oracle.

The cast of the normalised row back to the activation dtype is a rounding
decision taken in fp32 on the GPU and from a double value in the oracle; at
near-ties the two may land one ulp apart, which the weight multiply and its
own rounding can turn into two ulps of the normalised value.  The tests
therefore allow, per element, the effect of a two-ulp difference in the
normalised inputs, and bound the share of elements that need that allowance.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import F32_ATOL, MAG_REL, gpu_to_f64, host_f64, to_gpu, ulp_bf16

pytestmark = pytest.mark.gpu

GEN = lambda s: np.random.default_rng([91, s])  # noqa: E731


def _ulp(x, dtype):
    if dtype == "bf16":
        return ulp_bf16(x)
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 23)


def check_qk(got, x, w, eps, dtype, pos, inv, section, interleaved, orc, what):
    rot = 2 * len(inv)
    ref, mag, y = orc.qk_norm_mrope(x, w, eps, dtype, pos, inv, section, interleaved, with_mag=True)
    # pass-through channels: the normalised, weighted values
    # bf16: a rare one-ulp flip of the cast of xn moves xn * weight by up to
    # one ulp of y before its own rounding, so y itself by up to two ulps;
    # fp32: the fp32 mean and rsqrt against exact ones, a few ulps anywhere
    nulp = 2 if dtype == "bf16" else 4
    py, pg = y[..., rot:], got[..., rot:]
    dy = np.abs(pg - py)
    assert (dy <= nulp * _ulp(py, dtype)).all(), f"{what}: pass-through off by more than {nulp} ulp"
    flips = int((dy > 0).sum())
    # rotated channels: one ulp of the result, the cancellation floor, and the
    # effect of a one-ulp difference in either normalised input
    cos, sin = orc.mrope_cos_sin(pos, inv, section, interleaved)
    ya, yb = y[..., :rot // 2], y[..., rot // 2:rot]
    c, s = cos[:, None, :rot // 2], sin[:, None, :rot // 2]
    # out[j] = y[j] c - y[j+h] s ;  out[j+h] = y[j+h] c + y[j] s
    first = _ulp(ya, dtype) * np.abs(c) + _ulp(yb, dtype) * np.abs(s)
    second = _ulp(yb, dtype) * np.abs(c) + _ulp(ya, dtype) * np.abs(s)
    flip = nulp * np.concatenate([first, second], axis=-1)
    r, g = ref[..., :rot], got[..., :rot]
    err = np.abs(g - r)
    base = (_ulp(r, dtype) if dtype == "bf16" else F32_ATOL) + MAG_REL * mag
    assert (err <= base + flip).all(), f"{what}: rotated channel outside tolerance"
    beyond = int((err > base).sum())
    if dtype == "bf16":
        assert beyond <= max(4, 0.002 * err.size), f"{what}: {beyond} of {err.size} rotated values need the flip allowance"
        assert flips <= max(4, 0.002 * dy.size), f"{what}: {flips} of {dy.size} normalised values differ"
    return {"flips": flips, "beyond": beyond}


# (T, hq, hk, D, rot, section).  The library picks a lane layout by shape:
# rot < D with rot / 16 bytes a power of two takes rot / 16 bytes lanes per
# row (several chunks each); rot = D takes D / 32 bytes lanes (a chunk of
# each half); any other slice, one chunk per lane.  The cases reach all three.
CASES = [  # (T, hq, hk, D, rot, section)
    (37, 3, 2, 128, 64, (12, 10, 10)),
    (64, 24, 4, 256, 64, (11, 11, 10)),    # Qwen3.5 heads
    (33, 4, 4, 128, 128, (24, 20, 20)),    # full-dim rotary (Qwen3-Omni)
    (19, 2, 1, 64, 32, (6, 5, 5)),
    (8, 5, 3, 256, 256, (44, 42, 42)),
    (21, 3, 2, 128, 96, (16, 16, 16)),    # rotary slice of 12 (bf16) or 24 (fp32) chunks: one chunk per lane
    (29, 3, 2, 64, 64, (12, 10, 10)),     # whole-row slice of 64 channels: 4 (bf16) or 8 (fp32) lanes per row
    (23, 9, 3, 128, 128, (24, 20, 20)),   # 12 whole rows: three row groups in flight per warp (both dtypes)
    (17, 10, 2, 64, 64, (12, 10, 10)),    # 12 rows of 64: two groups in flight (bf16), three (fp32)
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_h%d_%d_D%d_r%d" % c[:5])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_qk_norm_mrope_small(case, dtype, orc):
    T, hq, hk, D, rot, section = case
    rng = GEN(T * 7 + D + rot)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q, k = gen(rng, (T, hq, D), 3.0), gen(rng, (T, hk, D), 3.0)
    wq, wk = gen(rng, (D,), 0.5), gen(rng, (D,), 0.5)
    p = rng.integers(0, 100000, (3, T)).astype(np.int32)
    inv = ipe.rope_inv_freq(rot, 1e6)
    oinv = orc.rope_inv_freq(rot, 1e6)
    gq, gk = to_gpu(q, dtype), to_gpu(k, dtype)
    if dtype == "f32" and D > 128:
        # a warp holds one head row as at most 32 chunks of 16 bytes: fp32
        # rows wider than 128 channels are a documented limit, refused on the
        # host before any launch, and q / k stay untouched
        with pytest.raises(ipe.IpeError) as e:
            ipe.qk_norm_mrope(gq, gk, to_gpu(wq, dtype), to_gpu(wk, dtype), torch.from_numpy(p).cuda(), inv,
                              section, True, eps=1e-6)
        assert e.value.status == ipe.IPE_ELIMIT, e.value
        assert np.array_equal(gpu_to_f64(gq), host_f64(q, dtype)) and np.array_equal(gpu_to_f64(gk), host_f64(k, dtype))
        return
    ipe.qk_norm_mrope(gq, gk, to_gpu(wq, dtype), to_gpu(wk, dtype), torch.from_numpy(p).cuda(), inv, section,
                      True, eps=1e-6)
    for nm, x, w, g in (("q", q, wq, gq), ("k", k, wk, gk)):
        check_qk(gpu_to_f64(g), host_f64(x, dtype), host_f64(w, dtype), 1e-6, dtype, p, oinv, section, True, orc,
                 f"{case} {dtype} {nm}")


LONG = [  # (T, hq, hk, D, rot, section, dtype, theta)
    # past the length where rows of four 16-byte chunks per lane take the
    # two-blocks-per-SM form; not a multiple of the warp count
    (16411, 5, 3, 256, 64, (11, 11, 10), "bf16", 1e7),
    # whole rows, several tokens per warp: two row groups in flight (bf16)
    # and three (fp32)
    (20011, 4, 4, 128, 128, (24, 20, 20), "bf16", 1e6),
    (12007, 9, 3, 128, 128, (24, 20, 20), "f32", 1e6),
]


@pytest.mark.parametrize("case", LONG, ids=lambda c: "T%d_h%d_%d_D%d_r%d" % c[:5])
def test_qk_norm_mrope_long_sequence(case, orc):
    # every token compared
    T, hq, hk, D, rot, section, dtype, theta = case
    rng = GEN(T)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q, k = gen(rng, (T, hq, D), 3.0), gen(rng, (T, hk, D), 3.0)
    wq, wk = gen(rng, (D,), 0.5), gen(rng, (D,), 0.5)
    p = rng.integers(0, 200000, (3, T)).astype(np.int32)
    gq, gk = to_gpu(q, dtype), to_gpu(k, dtype)
    ipe.qk_norm_mrope(gq, gk, to_gpu(wq, dtype), to_gpu(wk, dtype), torch.from_numpy(p).cuda(),
                      ipe.rope_inv_freq(rot, theta), section, True, eps=1e-6)
    oinv = orc.rope_inv_freq(rot, theta)
    for nm, x, w, g in (("q", q, wq, gq), ("k", k, wk, gk)):
        check_qk(gpu_to_f64(g), host_f64(x, dtype), host_f64(w, dtype), 1e-6, dtype, p, oinv, section, True, orc,
                 f"long {case[:5]} {nm}")


@pytest.mark.parametrize("name,layout", [("text_t4096_qwen35", "interleaved"), ("text_t32768_omni", "chunked"),
                                         ("prefill_t131072_video", "interleaved")])
def test_qk_norm_mrope_workload(name, layout, orc):
    w = wl.WORKLOADS[name]
    t = w.text
    inp = wl.text_inputs(w)
    rng = GEN(3)
    wq, wk = wl.normal_bf16(rng, (t.head_dim,), 0.5), wl.normal_bf16(rng, (t.head_dim,), 0.5)
    il = layout == "interleaved"
    gq, gk = to_gpu(inp["q"], "bf16"), to_gpu(inp["k"], "bf16")
    ipe.qk_norm_mrope(gq, gk, to_gpu(wq, "bf16"), to_gpu(wk, "bf16"), torch.from_numpy(inp["positions"]).cuda(),
                      ipe.rope_inv_freq(t.rot_dim, t.theta), t.section, il, eps=1e-6)
    sel = np.unique(np.concatenate([np.arange(64), np.arange(t.T - 64, t.T),
                                    np.random.default_rng(1).choice(t.T, 1024, replace=False)]))
    sel_t = torch.from_numpy(sel).cuda()
    oinv = orc.rope_inv_freq(t.rot_dim, t.theta)
    pos = inp["positions"][:, sel]
    for nm, x, wt, g in (("q", inp["q"], wq, gq), ("k", inp["k"], wk, gk)):
        check_qk(gpu_to_f64(g.index_select(0, sel_t)), host_f64(x[sel], "bf16"), host_f64(wt, "bf16"), 1e-6,
                 "bf16", pos, oinv, t.section, il, orc, f"{name} {nm}")


def test_qk_norm_rejects():
    q = torch.zeros(4, 2, 96, dtype=torch.bfloat16, device="cuda")    # 12 chunks: not a power of two
    w = torch.ones(96, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(3, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(ipe.IpeError) as e:
        ipe.qk_norm_mrope(q, None, w, w, pos, ipe.rope_inv_freq(32, 1e4), (6, 5, 5))
    assert e.value.status == ipe.IPE_ELIMIT
