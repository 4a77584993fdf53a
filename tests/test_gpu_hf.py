"""HF rounding mode (through the C ABI): bit for bit against the oracle's
emulation of the listings' rounding points, against a per-element statement
of the same rounding points (the interpolation), and against torch's own
arithmetic on the GPU (the rotation).

The interpolation has no transcendental step, so the oracle comparison is
exact.  The rotation's cos / sin are fp32 values of sincosf on the GPU and
correctly rounded values in the oracle; where the two differ by an fp32 ulp
the cast to bf16 can differ by one bf16 ulp, which the oracle comparison
allows (and counts).  Against torch, which evaluates cos / sin on the same
GPU, the comparison is exact.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import F32_ATOL, gpu_to_f64, host_f64, to_gpu, ulp_bf16
from pins import _interp_by_sample_points

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f32": torch.float32}

GRIDS = [
    ([(1, 4, 6), (2, 6, 4), (1, 48, 48), (1, 48, 64), (2, 28, 28), (1, 80, 56)], 2, 48),
    ([(1, 5, 7), (3, 1, 9), (1, 33, 17)], 1, 48),
    ([(1, 10, 14), (1, 64, 96)], 2, 32),
    # strips of more patches than the per-block plan holds (computed per row)
    ([(1, 4, 1100), (2, 2, 6)], 2, 48),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("grids,m,G", GRIDS, ids=["m2_g48", "m1_g48", "m2_g32", "m2_wide"])
def test_interp_hf_bitwise(dtype, grids, m, G, orc):
    rng = np.random.default_rng([G, m, len(grids)])
    C = 40 if dtype == "bf16" else 20
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    table = gen(rng, (G * G, C), 0.5)
    gt = to_gpu(table, dtype)
    got = ipe.vis_pos_interp(gt, grids, m, rounding="hf")
    ipe.device_status()
    want = orc.vis_pos_interp_hf(host_f64(table, dtype), grids, m, dtype)
    g = gpu_to_f64(got)
    assert g.shape == want.shape
    bad = np.argwhere(g != want)
    assert bad.size == 0, f"{len(bad)} values differ from the oracle, first at {bad[:4].tolist()}"
    # and the per-element statement of the same rounding points
    assert (g == _interp_by_sample_points(host_f64(table, dtype), grids, m, dtype)).all()


@pytest.mark.parametrize("name", ["vision_batch8_bf16", "prefill_t131072_video"])
def test_interp_hf_workloads(name, orc):
    w = wl.WORKLOADS[name]
    v = w.vision
    vin = wl.vision_inputs(w)
    gt = to_gpu(vin["table"], v.dtype)
    got = ipe.vis_pos_interp(gt, v.grid_thw, v.merge, rounding="hf")
    ipe.device_status()
    g = gpu_to_f64(got)
    assert (g == _interp_by_sample_points(host_f64(vin["table"], v.dtype), v.grid_thw, v.merge, v.dtype)).all()
    if name == "vision_batch8_bf16":
        want = orc.vis_pos_interp_hf(host_f64(vin["table"], v.dtype), v.grid_thw, v.merge, v.dtype)
        assert (g == want).all()


def _torch_rotation(x, cos, sin, rot):
    """(x_rot * cos) + (rotate_half(x_rot) * sin) in x's dtype, cos / sin
    [T, rot] fp32 cast to that dtype first; pass-through appended."""
    c = cos.to(x.dtype)[:, None, :]
    s = sin.to(x.dtype)[:, None, :]
    xr, xp = x[..., :rot], x[..., rot:]
    rh = torch.cat([-xr[..., rot // 2:], xr[..., :rot // 2]], dim=-1)
    return torch.cat([xr * c + rh * s, xp], dim=-1)


CASES = [  # (T, hq, hk, D, rot, section, dtype, stride_pad)
    (300, 24, 4, 256, 64, (11, 11, 10), "bf16", 0),
    (97, 8, 2, 128, 128, (24, 20, 20), "bf16", 0),
    (64, 4, 2, 64, 32, (6, 5, 5), "f32", 0),
    (45, 3, 1, 64, 64, (12, 10, 10), "bf16", 2),    # 4-byte token stride: the vector-load engine
    (40, 4, 2, 256, 256, (44, 42, 42), "bf16", 0),  # 128 frequencies: several 32-word rounds of the bf16 slot
]


def _case_tensors(case, seed):
    T, hq, hk, D, rot, section, dtype, pad = case
    rng = np.random.default_rng(seed)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q, k = gen(rng, (T, hq, D), 2.0), gen(rng, (T, hk, D), 2.0)

    def place(a, h):
        g = to_gpu(a, dtype)
        if not pad:
            return g
        buf = torch.zeros(T, h * D + pad, dtype=g.dtype, device="cuda")
        view = buf[:, :h * D].view(T, h, D)
        view.copy_(g)
        return view
    pos = rng.integers(0, 200000, (3, T)).astype(np.int32)
    return q, k, place(q, hq), place(k, hk), pos


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_h%d_%d_D%d_r%d_%s_pad%d" % (c[:5] + c[6:]))
def test_apply_rotary_partial_hf_matches_torch(case):
    # cos / sin tables given: the rounding sequence alone decides, bit for bit
    T, hq, hk, D, rot, section, dtype, pad = case
    q, k, gq, gk, pos = _case_tensors(case, 11)
    ang = torch.rand(T, rot // 2, device="cuda", generator=torch.Generator("cuda").manual_seed(3)) * 3000
    cos = torch.cat([ang.cos(), ang.cos()], -1).contiguous()
    sin = torch.cat([ang.sin(), ang.sin()], -1).contiguous()
    want_q, want_k = _torch_rotation(gq.clone(), cos, sin, rot), _torch_rotation(gk.clone(), cos, sin, rot)
    ipe.apply_rotary_partial(gq, gk, cos, sin, rounding="hf")
    ipe.device_status()
    assert torch.equal(gq, want_q) and torch.equal(gk, want_k)


@pytest.mark.parametrize("rot", [64, 128, 256])
def test_apply_rotary_partial_hf_unequal_halves(rot):
    # tables whose two halves differ (the literal formula reads cos / sin at
    # j + rot/2 for the second half): every coefficient array of the slot,
    # bit for bit against torch running the listing's steps
    T, hq, hk, D = 77, 5, 3, 256
    g = torch.Generator("cuda").manual_seed(rot)
    q = (torch.randn(T, hq, D, device="cuda", generator=g) * 2).to(torch.bfloat16)
    k = (torch.randn(T, hk, D, device="cuda", generator=g) * 2).to(torch.bfloat16)
    cos = torch.rand(T, rot, device="cuda", generator=g) * 2 - 1
    sin = torch.rand(T, rot, device="cuda", generator=g) * 2 - 1
    want_q, want_k = _torch_rotation(q.clone(), cos, sin, rot), _torch_rotation(k.clone(), cos, sin, rot)
    ipe.apply_rotary_partial(q, k, cos, sin, rounding="hf")
    ipe.device_status()
    assert torch.equal(q, want_q) and torch.equal(k, want_k)


def _torch_mrope_tables(pos, inv, section, interleaved, orc):
    """The listing's cos / sin on the GPU: fp32 position x inv_freq products,
    the per-frequency axis, cat(f, f), torch's cos and sin."""
    axis = torch.from_numpy(orc.mrope_axis_labels(len(inv), section, interleaved)).long().cuda()
    p = torch.from_numpy(pos).cuda().float()                          # [3, T]
    inv_t = torch.from_numpy(np.asarray(inv, np.float32)).cuda()
    freqs = p[:, :, None] * inv_t[None, None, :]                      # [3, T, half]
    f = freqs.gather(0, axis[None, None, :].expand(1, p.shape[1], -1))[0]
    emb = torch.cat([f, f], dim=-1)
    return emb.cos(), emb.sin()


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_h%d_%d_D%d_r%d_%s_pad%d" % (c[:5] + c[6:]))
@pytest.mark.parametrize("layout", ["interleaved", "chunked"])
def test_mrope_apply_hf(case, layout, orc):
    T, hq, hk, D, rot, section, dtype, pad = case
    il = layout == "interleaved"
    q, k, gq, gk, pos = _case_tensors(case, 12)
    inv = ipe.rope_inv_freq(rot, 1e6)
    cos, sin = _torch_mrope_tables(pos, inv, section, il, orc)
    want_q, want_k = _torch_rotation(gq.clone(), cos, sin, rot), _torch_rotation(gk.clone(), cos, sin, rot)
    ipe.mrope_apply(gq, gk, torch.from_numpy(pos).cuda(), inv, section, il, rounding="hf")
    ipe.device_status()
    # the same cos / sin as torch on this GPU, then the listing's roundings
    assert torch.equal(gq, want_q) and torch.equal(gk, want_k)
    # against the oracle (correctly rounded cos / sin): one-ulp casts may differ
    oinv = orc.rope_inv_freq(rot, 1e6)
    for nm, x, g in (("q", q, gq), ("k", k, gk)):
        xf = host_f64(x, dtype)
        ref = orc.mrope_apply_hf(xf, pos, oinv, section, il, dtype)
        got = gpu_to_f64(g)
        err = np.abs(got - ref)
        if dtype == "f32":
            assert err.max() <= F32_ATOL, f"{nm}: {err.max()}"
            continue
        c32, s32 = orc.mrope_cos_sin_f32(pos, oinv, section, il)
        h = rot // 2
        rh = np.concatenate([-xf[..., h:rot], xf[..., :h]], axis=-1)
        allow = np.abs(xf[..., :rot]) * ulp_bf16(c32)[:, None, :] + np.abs(rh) * ulp_bf16(s32)[:, None, :]
        tol = ulp_bf16(ref[..., :rot]) + 2 * allow
        assert (err[..., :rot] <= tol).all(), f"{nm}: beyond the cos / sin cast allowance"
        assert (err[..., rot:] == 0).all(), f"{nm}: pass-through changed"
        assert (err > 0).sum() <= max(8, 0.002 * err.size), f"{nm}: {(err > 0).sum()} values differ"


def test_sincos_matches_torch():
    # the fp32 cos / sin of the rotary kernels are those torch computes on the GPU
    T, rot = 4096, 64
    rng = np.random.default_rng(5)
    pos = rng.integers(0, 1 << 24, (3, T)).astype(np.int32)
    inv = ipe.rope_inv_freq(rot, 1e7)
    cos = torch.empty(T, rot, dtype=torch.float32, device="cuda")
    sin = torch.empty_like(cos)
    ipe.mrope_cos_sin(torch.from_numpy(pos).cuda(), inv, (11, 11, 10), False, cos, sin)
    ipe.device_status()
    import oracle
    tc, ts = _torch_mrope_tables(pos, inv, (11, 11, 10), False, oracle.get())
    assert torch.equal(cos, tc) and torch.equal(sin, ts)


def test_rounding_argument_rejected():
    q = torch.zeros(4, 1, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ipe.mrope_apply(q, None, torch.zeros(3, 4, dtype=torch.int32, device="cuda"), ipe.rope_inv_freq(64, 1e4),
                        (12, 10, 10), rounding="bf16")


def test_interp_hf_linspace_sweep():
    # Every grid side from 2 to 1024 (G = 48, merge 1): the HF kernel's sample
    # points are torch.linspace's fp32 points bit for bit, seen through the
    # blend of a random fp32 table (a point one ulp off changes its weights).
    rng = np.random.default_rng(77)
    table = wl.normal_f32(rng, (48 * 48, 8), 1.0)
    gt = to_gpu(table, "f32")
    sides = range(2, 1025)
    for grids in ([(1, n, 2) for n in sides], [(1, 2, n) for n in sides]):
        got = gpu_to_f64(ipe.vis_pos_interp(gt, grids, 1, rounding="hf"))
        want = _interp_by_sample_points(host_f64(table, "f32"), grids, 1, "f32")
        bad = np.argwhere(got != want)
        assert bad.size == 0, f"{len(bad)} values differ, first rows {bad[:4, 0].tolist()}"
