"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Indices, corner ids, (row, col) and axis maps are compared bit-exactly;
floating-point values with the tolerance model of ``gpu_helpers``.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import bf16_to_gpu, check, f32_to_gpu, gpu_to_f64, host_f64, to_gpu
from pins import golden

pytestmark = pytest.mark.gpu

GEN = lambda s: np.random.default_rng([77, s])  # noqa: E731 - small-case inputs


# ===================================================================== text


@pytest.mark.parametrize("half,section", [(32, (11, 11, 10)), (64, (24, 20, 20)), (10, (4, 3, 3)),
                                          (10, (6, 2, 2)), (2, (1, 1, 0)), (1, (1, 0, 0)), (64, (0, 32, 32)),
                                          (256, (100, 80, 76)), (7, (0, 0, 7))])
@pytest.mark.parametrize("interleaved", [True, False])
def test_axis_map_bitexact(half, section, interleaved, orc):
    got = ipe.mrope_axis_map(half, section, interleaved).cpu().numpy().astype(np.int64)
    assert np.array_equal(got, orc.mrope_axis_labels(half, section, interleaved))


def test_cos_sin_axis_reading_example():
    pos = torch.tensor([[1], [2], [3]], dtype=torch.int32, device="cuda")
    for key, vals in golden("axis_acos.txt"):
        sec, il = tuple(int(v) for v in key[:3]), int(key[3])
        cos, sin = ipe.mrope_cos_sin(pos, torch.ones(10), sec, bool(il))
        ang = np.rint(np.mod(np.arctan2(sin.cpu().numpy()[0], cos.cpu().numpy()[0]), 2 * np.pi)).astype(int)
        assert ang.tolist() == [int(v) for v in vals], (sec, il)


def test_rotary_worked_example_d4():
    g = {k[0]: np.array([float(v) for v in vals]) for k, vals in golden("rotary_d4.txt")}
    pos = torch.full((3, 1), 2, dtype=torch.int32, device="cuda")
    inv = torch.tensor([1.0, 0.01])
    cos, sin = ipe.mrope_cos_sin(pos, inv, (1, 1, 0), True)
    assert np.array_equal(np.round(cos.cpu().numpy()[0].astype(np.float64), 4), g["cos"])
    assert np.array_equal(np.round(sin.cpu().numpy()[0].astype(np.float64), 4), g["sin"])
    for i in (1, 2):
        x = f32_to_gpu(g[f"apply_in_{i}"].reshape(1, 1, 4))
        y = x.clone()
        ipe.apply_rotary_partial(x, None, cos, sin)
        assert np.array_equal(np.round(gpu_to_f64(x)[0, 0], 4) + 0.0, g[f"apply_out_{i}"])
        ipe.mrope_apply(y, None, pos, inv, (1, 1, 0), True)
        assert torch.equal(x, y)


def _rand_positions(rng, T, hi=200000):
    """Mixed text / vision-like positions."""
    p = rng.integers(0, hi, size=(3, T))
    text = rng.random(T) < 0.5
    p[1, text] = p[0, text]
    p[2, text] = p[0, text]
    return p.astype(np.int32)


SMALL = [  # (T, hq, hk, D, rot, section)
    (37, 3, 2, 48, 32, (6, 5, 5)),        # half 16: 8-wide bf16
    (50, 4, 1, 64, 64, (12, 10, 10)),     # full-dim rotary
    (19, 2, 2, 40, 24, (4, 4, 4)),        # half 12: 4-wide
    (23, 5, 3, 12, 4, (1, 1, 0)),         # half 2: 2-wide
    (31, 2, 1, 8, 2, (1, 0, 0)),          # half 1: scalar
    (1, 1, 1, 256, 64, (11, 11, 10)),
    (129, 24, 4, 256, 64, (11, 11, 10)),  # several tiles plus a ragged tail
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "T%d_h%d_%d_D%d_r%d" % c[:5])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("interleaved", [True, False])
def test_mrope_apply_small(case, dtype, interleaved, orc):
    T, hq, hk, D, rot, section = case
    rng = GEN(T * 1000 + D)
    pos = _rand_positions(rng, T)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q = gen(rng, (T, hq, D))
    k = gen(rng, (T, hk, D))
    inv = orc.rope_inv_freq(rot, 1e6)
    ginv = ipe.rope_inv_freq(rot, 1e6)
    gq, gk, gpos = to_gpu(q, dtype), to_gpu(k, dtype), torch.from_numpy(pos).cuda()
    fq, fk = gq.clone(), gk.clone()
    ipe.mrope_apply(fq, fk, gpos, ginv, section, interleaved)
    # unfused: the library's own tables, then the table rotation
    cos, sin = ipe.mrope_cos_sin(gpos, ginv, section, interleaved)
    ipe.apply_rotary_partial(gq, gk, cos, sin)
    assert torch.equal(fq, gq) and torch.equal(fk, gk), "fused and unfused differ"
    for name, x, g in (("q", q, fq), ("k", k, fk)):
        ref, mag = orc.mrope_apply(host_f64(x, dtype), pos, inv, section, interleaved, with_mag=True)
        out = gpu_to_f64(g)
        check(out[..., :rot], ref[..., :rot], mag, dtype, name)
        assert np.array_equal(out[..., rot:], host_f64(x, dtype)[..., rot:]), "pass-through changed"


@pytest.mark.parametrize("T,half,section", [(1000, 32, (11, 11, 10)), (777, 64, (24, 20, 20)),
                                             (1001, 256, (86, 85, 85)), (5, 12, (4, 4, 4)), (3, 3, (1, 1, 1))])
@pytest.mark.parametrize("interleaved", [True, False])
def test_cos_sin_tiles_and_tail(T, half, section, interleaved, orc):
    # the tables alone against the oracle: many tiles of tokens and a ragged
    # last one (tiles of 2048 / half tokens when half is a multiple of 4),
    # both halves of every row equal
    rng = GEN(T + half)
    pos = _rand_positions(rng, T)
    ginv = ipe.rope_inv_freq(2 * half, 1e6)
    cos, sin = ipe.mrope_cos_sin(torch.from_numpy(pos).cuda(), ginv, section, interleaved)
    rc, rs = orc.mrope_cos_sin(pos, orc.rope_inv_freq(2 * half, 1e6), section, interleaved)
    check(cos.cpu().numpy(), rc, None, "f32", "cos")
    check(sin.cpu().numpy(), rs, None, "f32", "sin")
    c = cos.cpu().numpy()
    assert np.array_equal(c[:, :half], c[:, half:])


def test_cos_sin_ulp_bound(orc):
    # The tables' sine / cosine (sincosf of the fp32 angle) against the
    # oracle's double values of the same angle: within 4 fp32 units in the
    # last place of the exact value (CUDA documents 2 for sinf and cosf),
    # over positions up to 2^24, where the angles of the lowest frequencies
    # take the large-argument reduction.  Each axis gets its own positions,
    # so every frequency sees large angles.
    T, half = 4096, 32
    rng = GEN(4242)
    pos = rng.integers(0, 1 << 23, size=(3, T))
    pos[:, :64] = rng.integers(1 << 23, 1 << 24, size=(3, 64))
    # integers next to multiples of pi/2: tiny reduced arguments
    k = rng.integers(1, 5_000_000, size=256)
    pos[0, 64:320] = np.rint(k * (np.pi / 2)).astype(np.int64)
    pos[:, 320:330] = np.arange(10)[None, :]
    pos = pos.astype(np.int32)
    inv = ipe.rope_inv_freq(2 * half, 1e6)
    for interleaved in (True, False):
        cos, sin = ipe.mrope_cos_sin(torch.from_numpy(pos).cuda(), inv, (11, 11, 10), interleaved)
        rc, rs = orc.mrope_cos_sin(pos, orc.rope_inv_freq(2 * half, 1e6), (11, 11, 10), interleaved)
        for name, got, ref in (("cos", cos.cpu().numpy(), rc), ("sin", sin.cpu().numpy(), rs)):
            ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
            err = np.abs(got.astype(np.float64) - ref) / ulp
            assert err.max() <= 4.0, (name, interleaved, float(err.max()), np.unravel_index(err.argmax(), err.shape))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_apply_rotary_partial_independent_tables(dtype, orc):
    # cos / sin are inputs: arbitrary tables whose halves differ exercise the
    # literal formula (cos[j + h], sin[j + h] on the second half).
    T, hq, hk, D, rot = 45, 6, 2, 80, 48
    rng = GEN(5)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q, k = gen(rng, (T, hq, D)), gen(rng, (T, hk, D))
    cos = rng.uniform(-1, 1, (T, rot)).astype(np.float32)
    sin = rng.uniform(-1, 1, (T, rot)).astype(np.float32)
    gq, gk = to_gpu(q, dtype), to_gpu(k, dtype)
    ipe.apply_rotary_partial(gq, gk, f32_to_gpu(cos), f32_to_gpu(sin))
    for name, x, g in (("q", q, gq), ("k", k, gk)):
        ref, mag = orc.apply_rotary(host_f64(x, dtype), cos.astype(np.float64), sin.astype(np.float64),
                                    with_mag=True)
        check(gpu_to_f64(g)[..., :rot], ref[..., :rot], mag, dtype, name)
        assert np.array_equal(gpu_to_f64(g)[..., rot:], host_f64(x, dtype)[..., rot:])


def test_text_only_layouts_bitwise_equal():
    T = 300
    p = np.arange(1000, 1000 + T, dtype=np.int32)
    pos = torch.from_numpy(np.stack([p, p, p])).cuda()
    inv = ipe.rope_inv_freq(64, 1e7)
    ci, si = ipe.mrope_cos_sin(pos, inv, (11, 11, 10), True)
    cc, sc = ipe.mrope_cos_sin(pos, inv, (11, 11, 10), False)
    c1, s1 = ipe.mrope_cos_sin(pos, inv, (32, 0, 0), True)
    assert torch.equal(ci, cc) and torch.equal(si, sc) and torch.equal(ci, c1) and torch.equal(si, s1)


def test_strided_fused_qkv_and_guards():
    # q and k as views of one fused qkv row [T, (hq + 2 hk) D]; v and the
    # guard rows must stay bit-identical.
    T, hq, hk, D, rot = 70, 8, 2, 128, 64
    rng = GEN(9)
    qkv = bf16_to_gpu(wl.normal_bf16(rng, (T + 2, (hq + 2 * hk) * D)))
    before = qkv.clone()
    body = qkv[1:T + 1]
    q = body[:, :hq * D].view(T, hq, D)
    k = body[:, hq * D:(hq + hk) * D].view(T, hk, D)
    pos = torch.from_numpy(_rand_positions(rng, T)).cuda()
    inv = ipe.rope_inv_freq(rot, 1e6)
    ipe.mrope_apply(q, k, pos, inv, (12, 10, 10), True)
    qc = before[1:T + 1, :hq * D].reshape(T, hq, D).clone()
    kc = before[1:T + 1, hq * D:(hq + hk) * D].reshape(T, hk, D).clone()
    ipe.mrope_apply(qc, kc, pos, inv, (12, 10, 10), True)
    assert torch.equal(q, qc) and torch.equal(k, kc)
    assert torch.equal(qkv[0], before[0]) and torch.equal(qkv[T + 1], before[T + 1])
    assert torch.equal(body[:, (hq + hk) * D:], before[1:T + 1, (hq + hk) * D:])
    assert torch.equal(body[:, :hq * D].view(T, hq, D)[..., rot:], before[1:T + 1, :hq * D].view(T, hq, D)[..., rot:])


def test_empty_and_single_tensor():
    inv = ipe.rope_inv_freq(64, 1e7)
    q = torch.zeros(0, 4, 256, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(3, 0, dtype=torch.int32, device="cuda")
    ipe.mrope_apply(q, None, pos, inv, (11, 11, 10))
    cos, sin = ipe.mrope_cos_sin(pos, inv, (11, 11, 10))
    assert cos.shape == (0, 64)
    k = bf16_to_gpu(wl.normal_bf16(GEN(1), (5, 2, 256)))
    k0 = k.clone()
    ipe.mrope_apply(None, k, torch.zeros(3, 5, dtype=torch.int32, device="cuda"), inv, (11, 11, 10))
    # position 0 is the identity rotation
    assert torch.equal(k, k0)


# -------------------------------------------------------- text workloads


def _text_case(name):
    w = wl.WORKLOADS[name]
    return w, wl.text_inputs(w)


def _sample_tokens(T, positions, n=2048, seed=0):
    """First and last tokens, every segment boundary and random ones."""
    rng = np.random.default_rng(seed)
    change = np.flatnonzero(np.any(np.diff(positions, axis=1) != 1, axis=0))
    pick = set(range(min(64, T))) | set(range(max(0, T - 64), T))
    for c in change[:512]:
        pick.update(range(max(0, c - 1), min(T, c + 3)))
    extra = rng.choice(T, size=min(T, max(0, n - len(pick))), replace=False)
    pick.update(int(e) for e in extra)
    return np.array(sorted(pick))


@pytest.mark.parametrize("name,layout", [("text_t4096_qwen35", "interleaved"),
                                         ("text_t32768_omni", "interleaved"),
                                         ("text_t32768_omni", "chunked"),
                                         ("prefill_t131072_video", "interleaved")])
def test_text_workload(name, layout, orc):
    w, inp = _text_case(name)
    t = w.text
    il = layout == "interleaved"
    pos = inp["positions"]
    inv = orc.rope_inv_freq(t.rot_dim, t.theta)
    gpos = torch.from_numpy(pos).cuda()
    ginv = ipe.rope_inv_freq(t.rot_dim, t.theta)
    gq, gk = bf16_to_gpu(inp["q"]), bf16_to_gpu(inp["k"])
    uq, uk = gq.clone(), gk.clone()
    ipe.mrope_apply(gq, gk, gpos, ginv, t.section, il)
    cos, sin = ipe.mrope_cos_sin(gpos, ginv, t.section, il)
    ipe.apply_rotary_partial(uq, uk, cos, sin)
    assert torch.equal(gq, uq) and torch.equal(gk, uk), "fused and unfused differ"
    sel = _sample_tokens(t.T, pos) if t.T > 40000 else np.arange(t.T)
    # cos / sin tables (fp32) on the sampled tokens
    rc, rs = orc.mrope_cos_sin(pos[:, sel], inv, t.section, il)
    check(cos.cpu().numpy()[sel], rc, None, "f32", "cos")
    check(sin.cpu().numpy()[sel], rs, None, "f32", "sin")
    sel_t = torch.from_numpy(sel).cuda()
    for nm, x, g in (("q", inp["q"], gq), ("k", inp["k"], gk)):
        ref, mag = orc.mrope_apply(host_f64(x[sel], "bf16"), pos[:, sel], inv, t.section, il, with_mag=True)
        out = gpu_to_f64(g.index_select(0, sel_t))
        check(out[..., :t.rot_dim], ref[..., :t.rot_dim], mag, "bf16", f"{name} {nm}")
        assert np.array_equal(out[..., t.rot_dim:], host_f64(x[sel], "bf16")[..., t.rot_dim:])


# =================================================================== vision

PLAN_GRIDS = [
    ([(1, 16, 16)], 2, 48), ([(1, 48, 48)], 2, 48), ([(2, 4, 6)], 2, 48), ([(1, 2, 2)], 2, 48),
    ([(1, 1, 5)], 1, 48), ([(1, 3, 1)], 1, 48), ([(1, 6, 9)], 3, 48), ([(1, 8, 12)], 2, 4),
    ([(1, 64, 96), (2, 28, 28), (1, 80, 56)], 2, 48), ([(16, 64, 64)], 2, 48),
    ([(1, 2, 4)] * 17 + [(3, 6, 2)], 2, 48),      # more than 16 images: the large descriptor
]


@pytest.mark.parametrize("grids,merge,G", PLAN_GRIDS, ids=lambda v: str(v)[:40])
def test_plan_bitexact(grids, merge, G, orc):
    idx4, w4, rowcol = ipe.vis_interp_plan(grids, merge, G)
    oidx, ow = orc.vis_interp_plan(grids, merge, G)
    assert np.array_equal(idx4.cpu().numpy().astype(np.int64), oidx)
    assert np.array_equal(rowcol.cpu().numpy().T.astype(np.int64), orc.vis_rot_pos_ids(grids, merge))
    # fp32 weights in [0, 1]: products of correctly rounded fractions
    assert np.abs(w4.cpu().numpy().astype(np.float64) - ow).max() <= 2.0 ** -22


def _vision_case(name):
    w = wl.WORKLOADS[name]
    return w, wl.vision_inputs(w)


def _interp_check(table, grids, merge, dtype, out, orc, what):
    ref, mag = orc.vis_pos_embed_interpolate(host_f64(table, dtype), grids, merge, with_mag=True)
    return check(gpu_to_f64(out), ref, mag, dtype, what)


@pytest.mark.parametrize("name", ["vision_16x16_f32", "vision_batch8_bf16", "prefill_t131072_video"])
def test_interp_workload(name, orc):
    w, inp = _vision_case(name)
    v = w.vision
    out = ipe.vis_pos_interp(to_gpu(inp["table"], v.dtype), v.grid_thw, v.merge)
    _interp_check(inp["table"], v.grid_thw, v.merge, v.dtype, out, orc, name)


@pytest.mark.parametrize("grids,merge,G,C", [
    ([(1, 48, 48)], 2, 48, 64), ([(1, 1, 5), (1, 3, 1)], 1, 48, 1152), ([(1, 6, 9)], 3, 48, 100),
    ([(1, 8, 12)], 2, 4, 36), ([(2, 4, 6), (1, 2, 2), (3, 6, 4)], 2, 48, 1000), ([(1, 2, 4)] * 20, 2, 48, 132),
    ([(1, 96, 2)], 2, 48, 1152), ([(1, 2, 1030), (1, 4, 4)], 2, 48, 64),   # wider than the column cache
    # enough strips for two channel slices per block, with a ragged last group
    ([(1, 24, 4)] * 100, 2, 48, 1000), ([(1, 12, 4)] * 400, 2, 48, 100), ([(1, 8, 4)] * 300, 1, 48, 1152)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_interp_edges(grids, merge, G, C, dtype, orc):
    rng = GEN(G * 7 + C)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    table = gen(rng, (G * G, C), 0.02)
    out = ipe.vis_pos_interp(to_gpu(table, dtype), grids, merge)
    _interp_check(table, grids, merge, dtype, out, orc, f"{grids} {dtype}")


def _rope_check(x, grids, merge, theta, dtype, g, orc, what, sample=None):
    pos_ids = orc.vis_rot_pos_ids(grids, merge)
    xs = host_f64(x, dtype)
    out = gpu_to_f64(g)
    if sample is not None:
        pos_ids, xs, out = pos_ids[sample], xs[sample], out[sample]
    cos, sin = orc.vis_rotary_cos_sin(pos_ids, xs.shape[2], theta)
    ref, mag = orc.apply_rotary(xs, cos, sin, with_mag=True)
    return check(out, ref, mag, dtype, what)


@pytest.mark.parametrize("name", ["vision_16x16_f32", "vision_batch8_bf16", "prefill_t131072_video"])
def test_vis_rope_workload(name, orc):
    w, inp = _vision_case(name)
    v = w.vision
    q, k = to_gpu(inp["q"], v.dtype), to_gpu(inp["k"], v.dtype)
    ipe.vis_rope2d(q, k, v.grid_thw, v.merge, v.theta)
    N = q.shape[0]
    sample = None
    if N > 30000:
        rng = np.random.default_rng(3)
        sample = np.unique(np.concatenate([np.arange(256), np.arange(N - 256, N),
                                           rng.choice(N, 4096, replace=False)]))
    _rope_check(inp["q"], v.grid_thw, v.merge, v.theta, v.dtype, q, orc, name + " q", sample)
    _rope_check(inp["k"], v.grid_thw, v.merge, v.theta, v.dtype, k, orc, name + " k", sample)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_vis_rope_edges(dtype, orc):
    rng = GEN(21)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    cases = [([(1, 2, 2)], 2, 3, 72), ([(2, 6, 4), (1, 4, 8)], 2, 5, 16), ([(1, 1, 7)], 1, 2, 8),
             ([(1, 6, 6)], 3, 1, 12), ([(1, 2, 2)] * 18, 2, 16, 72)]
    for grids, merge, heads, D in cases:
        N = sum(t * h * w for t, h, w in grids)
        x = gen(rng, (N, heads, D))
        g = to_gpu(x, dtype)
        ipe.vis_rope2d(g, None, grids, merge, 1e4)
        _rope_check(x, grids, merge, 1e4, dtype, g, orc, f"{grids} {D}")


def test_vis_rope_basis_readback(orc):
    grids = [(1, 4, 6)]
    pos = orc.vis_rot_pos_ids(grids, 2)
    inv = orc.rope_inv_freq(36, 1e4)
    x = np.zeros((24, 36, 72), np.float32)
    for j in range(36):
        x[:, j, j] = 1.0
    g = f32_to_gpu(x)
    ipe.vis_rope2d(g, None, grids, 2, 1e4)
    out = gpu_to_f64(g)
    for j in range(36):
        axis, i = (0, j) if j < 18 else (1, j - 18)
        a = (pos[:, axis].astype(np.float32) * inv[i]).astype(np.float64)
        assert np.abs(out[:, j, j] - np.cos(a)).max() <= 2e-7
        assert np.abs(out[:, j, j + 36] - np.sin(a)).max() <= 2e-7


def _frame_sample(grids, N, seed, n_random=4096, edge=256, around=8):
    """Patch rows for a sampled check at full size: both ends, a few rows on
    either side of every frame and image boundary, and random rows."""
    rows = [np.arange(min(edge, N)), np.arange(max(N - edge, 0), N)]
    r0 = 0
    for t, h, w in grids:
        for f in range(t + 1):
            b = r0 + f * h * w
            rows.append(np.arange(max(b - around, 0), min(b + around, N)))
        r0 += t * h * w
    rows.append(np.random.default_rng(seed).choice(N, min(n_random, N), replace=False))
    return np.unique(np.concatenate(rows))


@pytest.mark.parametrize("name", ["vision_batch8_bf16", "vision_16x16_f32", "prefill_t131072_video"])
def test_vis_fused_workload(name, orc):
    w, inp = _vision_case(name)
    v = w.vision
    table = to_gpu(inp["table"], v.dtype)
    q, k = to_gpu(inp["q"], v.dtype), to_gpu(inp["k"], v.dtype)
    q2, k2 = q.clone(), k.clone()
    out, _, _ = ipe.vis_pos_interp_rope2d(table, v.grid_thw, q, k, v.merge, v.theta)
    out2 = ipe.vis_pos_interp(table, v.grid_thw, v.merge)
    ipe.vis_rope2d(q2, k2, v.grid_thw, v.merge, v.theta)
    assert torch.equal(out, out2) and torch.equal(q, q2) and torch.equal(k, k2)
    # the interpolation is checked whole (the oracle blends a video's first
    # frame once and repeats it); the rotary on sampled rows at full size
    _interp_check(inp["table"], v.grid_thw, v.merge, v.dtype, out, orc, name)
    N = q.shape[0]
    sample = _frame_sample(v.grid_thw, N, seed=5) if N > 30000 else None
    _rope_check(inp["q"], v.grid_thw, v.merge, v.theta, v.dtype, q, orc, name + " q", sample)
    _rope_check(inp["k"], v.grid_thw, v.merge, v.theta, v.dtype, k, orc, name + " k", sample)


def test_interp_writes_nothing_outside_out():
    rng = GEN(4)
    table = bf16_to_gpu(wl.normal_bf16(rng, (48 * 48, 1152), 0.02))
    grids = [(2, 6, 8), (1, 4, 4)]
    N = 2 * 48 + 16
    buf = torch.full((N + 4, 1152), 7.0, dtype=torch.bfloat16, device="cuda")
    ipe.vis_pos_interp(table, grids, 2, out=buf[2:N + 2])
    assert (buf[:2] == 7.0).all() and (buf[N + 2:] == 7.0).all()
    assert not (buf[2:N + 2] == 7.0).all()


# ============================================================= host checks


def test_rejects_host_memory():
    # A pageable host pointer is rejected by the pointer-attribute check
    # before any launch.
    import ctypes
    inv = ipe.rope_inv_freq(64, 1e7)
    q = torch.zeros(16, 24, 256, dtype=torch.bfloat16)
    L = ipe.lib()
    sec = (ctypes.c_int32 * 3)(11, 11, 10)
    invh = (ctypes.c_float * 32)(*inv.tolist())
    pos = torch.zeros(3, 16, dtype=torch.int32, device="cuda")
    rc = L.ipe_mrope_apply(ctypes.c_void_p(q.data_ptr()), None, ipe.IPE_BF16, 16, 24, 0, 256, 6144, 0,
                           ctypes.c_void_p(pos.data_ptr()), invh, 64, sec, 1, None)
    assert rc == ipe.IPE_EINVAL and b"not device memory" in L.ipe_last_error()


def test_kernels_built_for_sm100a():
    # The CUDA runtime reports the architecture of the library's kernel code
    # as it loaded it on this device: sm_100a machine code.
    binary, ptx = ipe.kernel_arch()
    assert binary == 100, (binary, ptx)
    assert torch.cuda.get_device_capability() == (10, 0)


@pytest.mark.parametrize("grids,merge,C,heads,D", [
    ([(1, 48, 48)], 2, 64, 2, 72), ([(1, 1, 5), (1, 3, 1)], 1, 1152, 3, 16), ([(1, 6, 9)], 3, 100, 1, 12),
    ([(2, 4, 6), (1, 2, 2), (3, 6, 4)], 2, 1000, 4, 72), ([(1, 2, 4)] * 20, 2, 132, 2, 8),
    ([(1, 2, 1030), (1, 4, 4)], 2, 64, 1, 72), ([(1, 24, 4)] * 100, 2, 1000, 2, 16)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_vis_fused_edges(grids, merge, C, heads, D, dtype, orc):
    # the one-call entry on ragged shapes: the same interpolation and rotary
    # as the separate calls, bit for bit, and the oracle's values
    rng = GEN(C * 3 + D)
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    N = sum(t * h * w for t, h, w in grids)
    table = gen(rng, (48 * 48, C), 0.02)
    q, k = gen(rng, (N, heads, D)), gen(rng, (N, heads, D))
    gt, gq, gk = to_gpu(table, dtype), to_gpu(q, dtype), to_gpu(k, dtype)
    q2, k2 = gq.clone(), gk.clone()
    out, _, _ = ipe.vis_pos_interp_rope2d(gt, grids, gq, gk, merge, 1e4)
    out2 = ipe.vis_pos_interp(gt, grids, merge)
    ipe.vis_rope2d(q2, k2, grids, merge, 1e4)
    assert torch.equal(out, out2) and torch.equal(gq, q2) and torch.equal(gk, k2)
    _interp_check(table, grids, merge, dtype, out, orc, f"{grids} {dtype}")
    _rope_check(q, grids, merge, 1e4, dtype, gq, orc, f"{grids} {dtype} q")
