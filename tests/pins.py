"""Pins of the CPU oracle to facts fixed outside it.

Each pin takes an ``oracle.Oracle`` and raises ``AssertionError`` when the
oracle disagrees with a value printed on the pages (``tests/golden``), a closed
form, an invariant, a textbook special case or a brute-force statement.  The
same pins run against deliberately broken builds of the oracle
(``test_oracle_mutants.py``) to show that each plausible mistake is caught.
"""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    """Rows of a fixture: list of (key tokens, value tokens)."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, vals = line.partition(":")
            rows.append((key.split(), vals.split()))
    return rows


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------- text


def pin_inv_freq_golden(o):
    for key, vals in golden("inv_freq.txt"):
        dim, base, dec = int(key[0]), float(key[1]), int(key[2])
        got = np.round(o.rope_inv_freq(dim, base).astype(np.float64), dec)
        want = np.array([float(v) for v in vals])
        assert got.shape == want.shape and np.array_equal(got, want), (dim, base, got, want)


def pin_inv_freq_geometric(o):
    # The frequencies start at 1 and fall geometrically with ratio base^(2/dim)
    # ("Interleaved Rotary Position Embedding", RoPE section); fp32 rounding only.
    for dim, base in [(64, 1e7), (128, 1e6), (36, 1e4), (256, 1e4)]:
        inv = o.rope_inv_freq(dim, base).astype(np.float64)
        assert inv.shape == (dim // 2,)
        assert inv[0] == 1.0
        ratio = inv[1:] / inv[:-1]
        assert np.allclose(ratio, base ** (-2.0 / dim), rtol=3e-7, atol=0), (dim, base)
        assert abs(inv[-1] - base ** (-(dim - 2) / dim)) <= 6e-8 * inv[-1]


def pin_axis_acos_golden(o):
    pos = np.array([[1], [2], [3]])
    for key, vals in golden("axis_acos.txt"):
        sec, il = tuple(int(v) for v in key[:3]), int(key[3])
        cos, sin = o.mrope_cos_sin(pos, np.ones(10, np.float32), sec, il)
        got = np.rint(np.arccos(np.clip(cos[0], -1, 1))).astype(int)
        want = np.array([int(v) for v in vals])
        assert np.array_equal(got, want), (sec, il, got, want)
        # sin agrees with the same angle
        assert np.allclose(sin[0], np.sin(want), atol=1e-15)


def pin_axis_j7(o):
    for key, vals in golden("axis_j7.txt"):
        sec = tuple(int(v) for v in key)
        lab = o.mrope_axis_labels(10, sec, True)
        assert lab[7] == int(vals[0]), (sec, lab)


def pin_axis_qwen35(o):
    lab = o.mrope_axis_labels(32, (11, 11, 10), True)
    names = {"T": 0, "H": 1, "W": 2}
    seen = np.zeros(32, bool)
    for key, vals in golden("sections_qwen35.txt"):
        idx = [int(v) for v in vals]
        assert np.all(lab[idx] == names[key[0]]), (key, lab)
        seen[idx] = True
    assert seen.all()


def pin_axis_counts(o):
    # Each axis gets exactly its mrope_section share of frequencies, in both
    # layouts; chunked gives contiguous runs T..T H..H W..W.
    for half, sec in [(64, (24, 20, 20)), (32, (11, 11, 10)), (10, (4, 3, 3)), (10, (6, 2, 2)), (2, (1, 1, 0))]:
        for il in (True, False):
            lab = o.mrope_axis_labels(half, sec, il)
            assert [int((lab == a).sum()) for a in range(3)] == list(sec), (half, sec, il, lab)
        ch = o.mrope_axis_labels(half, sec, False)
        assert np.all(np.diff(ch) >= 0)
    # [24, 20, 20] interleaved: H at 1..58 step 3, W at 2..59 step 3, T elsewhere
    lab = o.mrope_axis_labels(64, (24, 20, 20), True)
    want = np.zeros(64, int)
    want[1:60:3] = 1
    want[2:60:3] = 2
    assert np.array_equal(lab, want)


def pin_rotary_d4_golden(o):
    g = {k[0]: np.array([float(v) for v in vals]) for k, vals in golden("rotary_d4.txt")}
    assert np.array_equal(o.rotate_half(g["rotate_half_in"]), g["rotate_half_out"])
    inv = np.array([1.0, 0.01], np.float32)
    pos = np.array([[2], [2], [2]])
    cos, sin = o.mrope_cos_sin(pos, inv, (1, 1, 0), True)
    assert np.array_equal(np.round(cos[0], 4), g["cos"]), cos
    assert np.array_equal(np.round(sin[0], 4), g["sin"]), sin
    for i in (1, 2):
        x = g[f"apply_in_{i}"].reshape(1, 1, 4)
        out = o.apply_rotary(x, cos, sin)[0, 0]
        assert np.array_equal(np.round(out, 4) + 0.0, g[f"apply_out_{i}"]), (i, out)


def pin_text_only_reduces_to_1d(o):
    # Text tokens (t = h = w): interleaved and chunked give bitwise the same
    # cos / sin, and the rotation is the textbook 1-D RoPE: pair (j, j + half)
    # is the complex number x_j + i x_{j+half} multiplied by exp(i p inv_j)
    # ("M01", step 5; "Interleaved Rotary Position Embedding", RoPE section).
    rng = _rng(7)
    half, sec = 32, (11, 11, 10)
    p = np.sort(rng.integers(0, 200000, 64))
    pos = np.stack([p, p, p])
    inv = o.rope_inv_freq(64, 1e7)
    ci, si = o.mrope_cos_sin(pos, inv, sec, True)
    cc, sc = o.mrope_cos_sin(pos, inv, sec, False)
    assert np.array_equal(ci, cc) and np.array_equal(si, sc)
    x = rng.standard_normal((64, 3, 96))
    out = o.apply_rotary(x, ci, si)
    ang = (p[:, None].astype(np.float32) * inv[None, :]).astype(np.float64)   # fp32 products
    z = (x[:, :, :half] + 1j * x[:, :, half:2 * half]) * np.exp(1j * ang)[:, None, :]
    assert np.allclose(out[:, :, :half], z.real, rtol=0, atol=1e-12)
    assert np.allclose(out[:, :, half:2 * half], z.imag, rtol=0, atol=1e-12)


def pin_rotation_invariants(o):
    rng = _rng(11)
    T, H, D, rot = 40, 5, 48, 32
    x = rng.standard_normal((T, H, D))
    pos = rng.integers(0, 5000, (3, T))
    inv = o.rope_inv_freq(rot, 1e4)
    cos, sin = o.mrope_cos_sin(pos, inv, (6, 5, 5), True)
    out = o.apply_rotary(x, cos, sin)
    h = rot // 2
    # channels >= rot pass through bit-identically
    assert np.array_equal(out[:, :, rot:], x[:, :, rot:])
    # every pair (j, j + rot/2) keeps its length
    n_in = x[:, :, :h] ** 2 + x[:, :, h:rot] ** 2
    n_out = out[:, :, :h] ** 2 + out[:, :, h:rot] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-13, atol=1e-13)


def pin_relative_position(o):
    # q(p) . k(p') depends only on p - p' (RoFormer property quoted on
    # "Interleaved Rotary Position Embedding", RoPE section).  Frequencies that
    # are powers of two keep every fp32 angle exact, so the check is exact.
    rng = _rng(3)
    half = 8
    inv = (2.0 ** -np.arange(half)).astype(np.float32)
    q = rng.standard_normal((1, 1, 2 * half))
    k = rng.standard_normal((1, 1, 2 * half))

    def rot(x, p):
        pos = np.array([[p], [p], [p]])
        c, s = o.mrope_cos_sin(pos, inv, (half, 0, 0), True)
        return o.apply_rotary(x, c, s)[0, 0]

    for p, pk, shift in [(5, 2, 17), (100, 300, 1000), (0, 9, 4096)]:
        d0 = rot(q, p) @ rot(k, pk)
        d1 = rot(q, p + shift) @ rot(k, pk + shift)
        assert abs(d0 - d1) < 1e-11, (p, pk, shift, d0, d1)


def pin_vision_tokens_per_axis(o):
    # A vision token's rotary angle at frequency j is the selected axis
    # position times inv_j: [2, 3, 4] for I12 gives 2,3,4,2,3,4,... under
    # [11, 11, 10] ("Interleaved Rotary Position Embedding", I12 example).
    inv = np.ones(32, np.float32)
    cos, sin = o.mrope_cos_sin(np.array([[2], [3], [4]]), inv, (11, 11, 10), True)
    ang = np.rint(np.mod(np.arctan2(sin[0, :32], cos[0, :32]), 2 * np.pi)).astype(int)
    want = np.array([[2, 3, 4][j % 3] for j in range(32)])
    assert np.array_equal(ang, want), ang
    assert np.array_equal(cos[0, 32:], cos[0, :32])


def pin_rms_norm_golden(o):
    g = {k[0]: np.array([float(v) for v in vals]) for k, vals in golden("rms_norm.txt")}
    out = o.rms_norm(g["x"].reshape(2, 2), g["weight"], 0.0, "f32")
    assert np.array_equal(np.round(out.reshape(-1), 4), g["out"]), out


def pin_rms_norm_closed_forms(o):
    # eps sits inside the square root: x = [1, 1], eps = 3 -> 1 / sqrt(1 + 3) = 0.5
    out = o.rms_norm(np.array([[1.0, 1.0]]), np.array([1.0, 3.0]), 3.0, "f32")
    assert np.array_equal(out, [[0.5, 1.5]])
    # a zero row with eps > 0 stays zero; with unit weight the row RMS is 1
    assert not o.rms_norm(np.zeros((1, 8)), np.ones(8), 1e-6, "f32").any()
    rng = _rng(17)
    x = rng.standard_normal((16, 64))
    y = o.rms_norm(x, np.ones(64), 0.0, "f32")
    assert np.allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=0, atol=2e-7)
    # scale invariance, and the bf16 result is bf16-representable
    y2 = o.rms_norm(7.25 * x, np.ones(64), 0.0, "f32")
    assert np.allclose(y, y2, rtol=2 ** -22, atol=0)
    yb = o.rms_norm(x, np.full(64, 1.5), 1e-6, "bf16").astype(np.float32)
    assert not (yb.view(np.uint32) & 0xFFFF).any()


def pin_rms_norm_matches_torch_literal(o):
    # The drill's steps evaluated by torch on the CPU in bf16: x.float(),
    # rsqrt(mean(x^2) + eps), .to(bf16), then * weight (a bf16 product).
    # The oracle (double, then the two roundings) agrees with it except at
    # rare fp32-vs-double ties; multiplying by the weight before the cast
    # agrees on only about three quarters of the elements.
    import torch
    rng = _rng(41)
    x = torch.from_numpy(rng.standard_normal((192, 128)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((1 + 0.3 * rng.standard_normal(128)).astype(np.float32)).to(torch.bfloat16)
    x32 = x.float()
    xn = x32 * torch.rsqrt(x32.pow(2).mean(-1, keepdim=True) + 1e-6)
    want = (xn.to(torch.bfloat16) * w).float().numpy().astype(np.float64)
    got = o.rms_norm(x.float().numpy().astype(np.float64), w.float().numpy().astype(np.float64), 1e-6, "bf16")
    assert (got == want).mean() >= 0.999


# ------------------------------------------------------------------- vision


def _merge_order_rowcol(t, h, w, m):
    """Brute-force statement of the output order: merge-block row, merge-block
    column, then the m x m patches inside, for each frame ("cortiq-engine
    qwen3vis.rs", positions() and rope_angles() loops)."""
    out = []
    for _ in range(t):
        for by in range(h // m):
            for bx in range(w // m):
                for iy in range(m):
                    for ix in range(m):
                        out.append((by * m + iy, bx * m + ix))
    return np.array(out, np.int64).reshape(-1, 2)


def pin_patch_counts(o):
    g = {k[0]: [int(v) for v in vals] for k, vals in golden("patch_counts.txt")}
    assert o.grid_patches(g["grid_thw"], 2) == g["patches"][0]
    assert o.grid_patches(g["grid_thw"], 2) // 4 == g["merged_tokens"][0]
    assert o.vis_rot_pos_ids(g["grid_thw"], 2).shape == (3072, 2)


def pin_exact_lookup_48(o):
    # h = w = G: every sample lands on a grid point, weights (1, 0, 0, 0), and
    # the output is the table itself in merge order.
    rng = _rng(5)
    G, C = 48, 24
    table = rng.standard_normal((G * G, C))
    out = o.vis_pos_embed_interpolate(table, [(1, 48, 48)], 2)
    rc = _merge_order_rowcol(1, 48, 48, 2)
    assert np.array_equal(out, table[rc[:, 0] * G + rc[:, 1]])
    idx, w = o.vis_interp_plan([(1, 48, 48)], 2, G)
    assert np.array_equal(w[0], np.ones(48 * 48)) and not w[1:].any()
    assert np.array_equal(idx[0], rc[:, 0] * G + rc[:, 1])


def pin_bilinear_reproduces_bilinear_functions(o):
    # Bilinear interpolation reproduces a + b y + c x + d x y exactly, sampled
    # at y = row (G-1)/(h-1), x = col (G-1)/(w-1) (0 when the side is 1).
    G = 48
    gy, gx = np.meshgrid(np.arange(G, dtype=np.float64), np.arange(G, dtype=np.float64), indexing="ij")
    coef = [(0.5, -1.25, 2.0, 0.0), (0.1, 0.0, 0.0, 0.03), (-2.0, 0.7, -0.3, 0.011)]
    table = np.stack([a + b * gy + c * gx + d * gx * gy for a, b, c, d in coef], -1).reshape(G * G, -1)
    for grid, m in [((1, 16, 16), 2), ((1, 32, 48), 2), ((2, 28, 28), 2), ((1, 64, 96), 2),
                    ((1, 80, 56), 2), ((1, 1, 5), 1), ((1, 3, 1), 1), ((1, 6, 9), 3)]:
        t, h, w = grid
        out = o.vis_pos_embed_interpolate(table, [grid], m)
        rc = _merge_order_rowcol(t, h, w, m)
        y = rc[:, 0] * (G - 1) / (h - 1) if h > 1 else np.zeros(len(rc))
        x = rc[:, 1] * (G - 1) / (w - 1) if w > 1 else np.zeros(len(rc))
        want = np.stack([a + b * y + c * x + d * x * y for a, b, c, d in coef], -1)
        assert np.allclose(out, want, rtol=0, atol=1e-12), grid


def pin_interp_weights(o):
    for grid in [(1, 16, 16), (1, 32, 48), (2, 28, 28), (1, 80, 56), (1, 2, 2)]:
        idx, w = o.vis_interp_plan([grid], 2, 48)
        assert np.allclose(w.sum(0), 1.0, rtol=0, atol=1e-15)
        assert (w >= 0).all() and (w <= 1).all()
        assert (idx >= 0).all() and (idx < 48 * 48).all()
        # corners share rows / columns: TL, TR on one row; TL, BL in one column
        assert np.array_equal(idx[0] // 48, idx[1] // 48) and np.array_equal(idx[2] // 48, idx[3] // 48)
        assert np.array_equal(idx[0] % 48, idx[2] % 48) and np.array_equal(idx[1] % 48, idx[3] % 48)


def pin_frames_and_concat(o):
    # t frames repeat the same image; images concatenate in grid_thw order.
    rng = _rng(9)
    table = rng.standard_normal((48 * 48, 8))
    grids = [(2, 4, 6), (1, 2, 2), (3, 6, 4)]
    out = o.vis_pos_embed_interpolate(table, grids, 2)
    off = 0
    for t, h, w in grids:
        single = o.vis_pos_embed_interpolate(table, [(1, h, w)], 2)
        for f in range(t):
            assert np.array_equal(out[off + f * h * w: off + (f + 1) * h * w], single)
        off += t * h * w
    assert off == out.shape[0]


def pin_merge_order_brute_force(o):
    # The 6-D permute of the interpolation, the broadcast of rot_pos_emb and a
    # brute-force loop all give the same (row, col) order.
    G = 48
    gy, gx = np.meshgrid(np.arange(G), np.arange(G), indexing="ij")
    # a table whose rows encode their own (row, col) grid point
    table = np.stack([gy, gx], -1).reshape(G * G, 2).astype(np.float64)
    for grid in [(1, 2, 2), (1, 4, 6), (2, 6, 4), (1, 2, 8), (2, 8, 2)]:
        t, h, w = grid
        rc = _merge_order_rowcol(t, h, w, 2)
        assert np.array_equal(o.vis_rot_pos_ids([grid], 2), rc)
    for grid in [(1, 48, 48), (2, 48, 48)]:
        out = o.vis_pos_embed_interpolate(table, [grid], 2)
        assert np.array_equal(out.astype(np.int64), _merge_order_rowcol(*grid, 2))


def pin_vision_angles_basis(o):
    # Reading the angles back: q = e_j gives (cos a_j, sin a_j) in channels
    # (j, j + 36); a_j is row * inv_j for j < 18 and col * inv_(j-18) after
    # ("cortiq-engine qwen3vis.rs", rope_angles() and attention()).
    grid = [(1, 4, 6)]
    pos = o.vis_rot_pos_ids(grid, 2)
    N, D = pos.shape[0], 72
    inv = o.rope_inv_freq(36, 1e4)
    for j in [0, 5, 17, 18, 23, 35]:
        x = np.zeros((N, 1, D))
        x[:, 0, j] = 1.0
        out = o.vis_apply_rotary(x, grid, 2, 1e4)[:, 0]
        axis, i = (0, j) if j < 18 else (1, j - 18)
        a = (pos[:, axis].astype(np.float32) * inv[i]).astype(np.float64)
        assert np.allclose(out[:, j], np.cos(a), atol=1e-15)
        assert np.allclose(out[:, j + 36], np.sin(a), atol=1e-15)
        others = np.delete(out, [j, j + 36], axis=1)
        assert not others.any()


def _patch_rowcol(grids, m):
    """(row, col) of every output row from its index alone.  Inside a frame,
    patch q = r mod (h w) is patch q mod m^2 (row-major, m x m) of merge
    block q div m^2, and the blocks run row-major over the (h/m) x (w/m)
    block grid; frames repeat and images follow one another."""
    out = []
    for t, h, w in grids:
        q = np.arange(t * h * w) % (h * w)
        blk, inner = q // (m * m), q % (m * m)
        by, bx = blk // (w // m), blk % (w // m)
        out.append(np.stack([by * m + inner // m, bx * m + inner % m], 1))
    return np.concatenate(out).astype(np.int64)


def _vision_rotary_fp32(q, grids, m, theta):
    """The vision rotary evaluated in fp32 from its definition: channel pair
    (j, j + D/2) of every head turns by a_j, with a_j = row * w_j for
    j < D/4 and col * w_(j - D/4) above, w_i = theta^(-2i / (D/2)) (formed
    here as exp(-(2i / (D/2)) ln theta) in fp32), and (row, col) the patch's
    grid point in merge order."""
    N, H, D = q.shape
    rc = _patch_rowcol(grids, m).astype(np.float32)
    i = np.arange(D // 4, dtype=np.float32)
    w = np.exp(-(np.float32(2) * i / np.float32(D // 2)) * np.float32(np.log(theta)))
    ang = np.concatenate([rc[:, :1] * w[None], rc[:, 1:] * w[None]], 1)          # [N, D/2] fp32
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = q[..., :D // 2].astype(np.float32), q[..., D // 2:].astype(np.float32)
    return np.concatenate([a * c - b * s, b * c + a * s], -1).astype(np.float64)


def pin_patch_rowcol_closed_form(o):
    # the closed form of the merge order against the brute-force loops
    for grids, m in [([(1, 4, 6), (2, 6, 4), (1, 8, 8)], 2), ([(3, 6, 9)], 3), ([(1, 1, 5), (2, 3, 1)], 1)]:
        brute = np.concatenate([_merge_order_rowcol(t, h, w, m) for t, h, w in grids])
        assert np.array_equal(_patch_rowcol(grids, m), brute)
        assert np.array_equal(o.vis_rot_pos_ids(grids, m), brute)


def pin_vision_rotary_matches_fp32_angles(o):
    # fp32 evaluation of the definition against the double oracle: agreement
    # to fp32 rounding (angles up to 7 rad, so a few 1e-6)
    rng = _rng(43)
    grids = [(1, 4, 6), (2, 6, 4), (1, 8, 8)]
    N = sum(t * h * w for t, h, w in grids)
    q = rng.standard_normal((N, 3, 72)).astype(np.float32)
    want = _vision_rotary_fp32(q, grids, 2, 1e4)
    got = o.vis_apply_rotary(q.astype(np.float64), grids, 2, 1e4)
    assert np.abs(got - want).max() <= 2e-5, np.abs(got - want).max()


def pin_vision_rotation_complex(o):
    # Whole-head split-half rotation = complex multiply of x_j + i x_(j+36)
    # by exp(i a_j); norm of every pair preserved.
    rng = _rng(13)
    grid = [(2, 4, 4)]
    pos = o.vis_rot_pos_ids(grid, 2)
    N = pos.shape[0]
    x = rng.standard_normal((N, 3, 72))
    out = o.vis_apply_rotary(x, grid, 2, 1e4)
    inv = o.rope_inv_freq(36, 1e4)
    a = np.concatenate([(pos[:, :1].astype(np.float32) * inv[None, :]),
                        (pos[:, 1:].astype(np.float32) * inv[None, :])], 1).astype(np.float64)
    z = (x[:, :, :36] + 1j * x[:, :, 36:]) * np.exp(1j * a)[:, None, :]
    assert np.allclose(out[:, :, :36], z.real, rtol=0, atol=1e-12)
    assert np.allclose(out[:, :, 36:], z.imag, rtol=0, atol=1e-12)


# -------------------------------------------------------- position table


def _l10_example():
    # t0, S, six merged slots of a [1, 4, 6] image (m = 2), E, t1
    return [0, 0, 1, 1, 1, 1, 1, 1, 0, 0], [[1, 4, 6]]


def pin_rope_index_golden(o):
    want = {k[0]: [int(v) for v in vals] for k, vals in golden("positions_l10.txt")}
    types, grids = _l10_example()
    pos, deltas = o.rope_index([types], None, grids, None, 2)
    for a, key in enumerate("THW"):
        assert pos[a, 0].tolist() == want[key], key
    # the next rotary position (7) minus the 10 kept slots
    assert deltas.tolist() == [-3]


def pin_rope_index_padding(o):
    # Padded slots (mask 0) are dropped before the runs are formed and keep
    # position 0; a masked slot inside the image run does not split it.
    types, grids = _l10_example()
    want, wd = o.rope_index([types], None, grids, None, 2)
    for left, right in [(3, 0), (0, 4), (2, 2)]:
        L = left + len(types) + right
        ty = [0] * left + types + [2] * right
        mk = [0] * left + [1] * len(types) + [0] * right
        pos, deltas = o.rope_index([ty], [mk], grids, None, 2)
        assert (pos[:, 0, left:left + len(types)] == want[:, 0]).all()
        assert not pos[:, 0, :left].any() and not pos[:, 0, left + len(types):].any()
        assert deltas.tolist() == wd.tolist() and pos.shape == (3, 1, L)
    ty = types[:5] + [0] + types[5:]
    mk = [1] * 5 + [0] + [1] * 5
    pos, _ = o.rope_index([ty], [mk], grids, None, 2)
    assert (np.delete(pos[:, 0], 5, axis=1) == want[:, 0]).all() and not pos[:, 0, 5].any()


def _random_batch(rng, B, merge=2):
    """Types, mask and grids of B mixed sequences: text, images, video slices
    each behind a timestamp token, audio; random left or right padding."""
    seqs, img, vid = [], [], []
    for _ in range(B):
        ty = []
        for _ in range(rng.integers(1, 6)):
            ty += [0] * int(rng.integers(1, 4))
            kind = rng.integers(0, 4)
            if kind == 1:
                t, h, w = int(rng.integers(1, 3)), 2 * int(rng.integers(1, 5)), 2 * int(rng.integers(1, 5))
                img.append([t, h, w])
                ty += [1] * (t * (h // merge) * (w // merge))
            elif kind == 2:
                t, h, w = int(rng.integers(1, 4)), 2 * int(rng.integers(1, 5)), 2 * int(rng.integers(1, 5))
                vid.append([t, h, w])
                for _ in range(t):
                    ty += [0] * int(rng.integers(1, 3)) + [2] * ((h // merge) * (w // merge))
            elif kind == 3:
                ty += [3] * int(rng.integers(1, 5))
        seqs.append(ty)
    L = max(len(t) for t in seqs) + 3
    types = np.zeros((B, L), np.int64)
    mask = np.zeros((B, L), np.int64)
    for b, ty in enumerate(seqs):
        off = int(rng.integers(0, L - len(ty) + 1))
        types[b, off:off + len(ty)] = ty
        types[b, :off] = rng.integers(0, 3, off)
        mask[b, off:off + len(ty)] = 1
    return types, mask, np.array(img, np.int64).reshape(-1, 3), np.array(vid, np.int64).reshape(-1, 3)


def _rope_index_prefix_form(types, mask, img, vid, m):
    """The same table from running counts instead of runs: a text slot sits
    at (kept text slots before it) + (advances of the vision runs before it);
    a vision run starts there and lays its grid out width-fastest."""
    slices = [(1, h, w) for t, h, w in vid for _ in range(t)]
    grids = {1: iter([tuple(g) for g in img]), 2: iter(slices)}
    B, L = types.shape
    pos = np.zeros((3, B, L), np.int64)
    deltas = np.zeros(B, np.int64)
    for b in range(B):
        text_before, vision_adv, prev, hi, n = 0, 0, None, None, 0
        for l in range(L):
            if not mask[b, l]:
                continue
            ty = int(types[b, l])
            if ty in (0, 3):
                pos[:, b, l] = text_before + vision_adv
                text_before += 1
            else:
                if ty != prev:
                    t, h, w = next(grids[ty])
                    start, off, gh, gw = text_before + vision_adv, 0, h // m, w // m
                    vision_adv += max(h, w) // m
                tt, rem = divmod(off, gh * gw)
                pos[:, b, l] = (start + tt, start + rem // gw, start + rem % gw)
                off += 1
            prev = ty
            n += 1
            hi = pos[:, b, l].max() if hi is None else max(hi, pos[:, b, l].max())
        deltas[b] = 0 if n == 0 else hi + 1 - n
    return pos, deltas


def pin_rope_index_prefix_form(o):
    rng = _rng(17)
    for B in (1, 3, 6):
        types, mask, img, vid = _random_batch(rng, B)
        pos, deltas = o.rope_index(types, mask, img, vid, 2)
        want, wd = _rope_index_prefix_form(types, mask, img, vid, 2)
        assert (pos == want).all() and (deltas == wd).all()
    # text only: arange on all three rows, delta 0
    pos, deltas = o.rope_index(np.zeros((2, 7), np.int64), None, None, None, 2)
    assert (pos == np.arange(7)[None, None, :]).all() and not deltas.any()


def pin_rope_index_errors(o):
    types, grids = _l10_example()
    for args in [([types], None, None, None, 2),                      # no image grid left
                 ([types], None, [[1, 4, 4]], None, 2),               # 4 slots for a 6-slot run
                 ([[0, 2, 2, 0, 2, 2]], None, None, [[1, 2, 4]], 2)]:  # one slice, two runs
        try:
            o.rope_index(*args)
        except ValueError:
            continue
        raise AssertionError(f"accepted {args}")


def pin_decode_continues_prefill(o):
    # The delta saved at prefill is the next rotary position minus the kept
    # length, so the first generated token lands one past the largest prefill
    # coordinate on all three axes.
    rng = _rng(23)
    types, mask, img, vid = _random_batch(rng, 5)
    pos, deltas = o.rope_index(types, mask, img, vid, 2)
    grown = np.concatenate([mask, np.ones((mask.shape[0], 1), np.int64)], axis=1)
    nxt = o.decode_positions(1, mask=grown, deltas=deltas)[:, :, 0]
    for b in range(types.shape[0]):
        top = pos[:, b][:, mask[b] == 1].max()
        assert (nxt[:, b] == top + 1).all(), (b, nxt[:, b], top)
    # the same from cache lengths (no padding): the kept length is the cache length
    nxt2 = o.decode_positions(1, cache_len=mask.sum(1), deltas=deltas)[:, :, 0]
    assert (nxt2 == nxt).all()


def pin_decode_closed_forms(o):
    # cache lengths: arange from the length, plus the delta, on all rows
    got = o.decode_positions(3, cache_len=[5, 0], deltas=[-2, 7])
    assert (got == np.array([[3, 4, 5], [7, 8, 9]])[None]).all()
    # mask with left padding: the sequence index counts kept slots only
    mask = [[0, 0, 1, 1, 1], [1, 1, 1, 1, 1]]
    got = o.decode_positions(2, mask=mask, deltas=[0, 10])
    assert (got == np.array([[1, 2], [13, 14]])[None]).all()
    # a padded new slot sits at 0 before the delta
    got = o.decode_positions(1, mask=[[1, 1, 0]], deltas=[4])
    assert (got[:, 0, 0] == 4).all()


# ------------------------------------------------------------ HF rounding


def _round_to(x, dtype):
    """fp32 values rounded to the dtype (nearest, ties to even); fp32 as is."""
    x = np.asarray(x, np.float32)
    if dtype == "bf16":
        import workloads as wl
        return wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x))
    return x


def _interp_by_sample_points(table, grids, m, rounding):
    """Every output row as the bilinear blend of the table at its own sample
    point.  The point of grid row i of an n-row image is the fp32
    torch.linspace(0, G-1, n)[i] (torch's own routine, which fixes the HF
    sample points); its corners are the floor y0 and min(y0 + 1, G - 1), its
    fraction f = point - y0, and the four weights (1-fy)(1-fx), (1-fy)fx,
    fy(1-fx), fy fx are fp32 products, in the corner order TL, TR, BL, BR.
      rounding "f64":  weights widened to double, blend in double;
      "f32" / "bf16":  the HF rounding points -- each weight rounded to the
                       dtype, each weight x value product and each partial
                       sum, taken left to right over the corners, computed
                       in fp32 and rounded to the dtype.
    table: [G*G, C] float64 holding values of the dtype.  Frames repeat
    their image; rows are in merge order."""
    import torch
    G = int(round(table.shape[0] ** 0.5))
    out = []
    for t, h, w in grids:
        rc = _patch_rowcol([(1, h, w)], m)
        sy = torch.linspace(0, G - 1, h).numpy()[rc[:, 0]]
        sx = torch.linspace(0, G - 1, w).numpy()[rc[:, 1]]
        y0, x0 = np.floor(sy).astype(np.int64), np.floor(sx).astype(np.int64)
        y1, x1 = np.minimum(y0 + 1, G - 1), np.minimum(x0 + 1, G - 1)
        fy, fx = sy - y0.astype(np.float32), sx - x0.astype(np.float32)
        one = np.float32(1)
        weights = [(one - fy) * (one - fx), (one - fy) * fx, fy * (one - fx), fy * fx]
        corners = [y0 * G + x0, y0 * G + x1, y1 * G + x0, y1 * G + x1]
        if rounding == "f64":
            frame = sum(wt.astype(np.float64)[:, None] * table[c] for wt, c in zip(weights, corners))
        else:
            frame = None
            for wt, c in zip(weights, corners):
                p = _round_to(_round_to(wt, rounding)[:, None] * table[c].astype(np.float32), rounding)
                frame = p if frame is None else _round_to(frame + p, rounding)
            frame = frame.astype(np.float64)
        out.append(np.tile(frame, (t, 1)))
    return np.concatenate(out)


def pin_interp_hf_matches_sample_points(o):
    # The oracle's HF mode (the listing's tensor steps, in C) against the
    # per-element statement above, bit for bit
    rng = _rng(29)
    cases = [([(1, 4, 6), (2, 6, 4), (1, 48, 48), (1, 10, 14)], 2), ([(1, 5, 7), (3, 1, 9)], 1)]
    for dt in ("bf16", "f32"):
        vals = _round_to(rng.standard_normal((48 * 48, 24)), dt).astype(np.float64)
        for grids, m in cases:
            want = _interp_by_sample_points(vals, grids, m, dt)
            got = o.vis_pos_interp_hf(vals, grids, m, dt)
            assert got.shape == want.shape and (got == want).all(), (dt, grids)


def pin_interp_matches_sample_points(o):
    # The default interpolation (exact sample points, double) against the
    # per-element blend at the fp32 linspace points: they differ only by the
    # rounding of the sample points (a few 1e-7 of a table value).
    rng = _rng(47)
    table = rng.standard_normal((48 * 48, 12))
    for grids, m in [([(1, 4, 6), (2, 10, 14), (1, 48, 64)], 2), ([(1, 5, 7), (3, 1, 9)], 1)]:
        want = _interp_by_sample_points(table, grids, m, "f64")
        got = o.vis_pos_embed_interpolate(table, grids, m)
        assert np.abs(got - want).max() <= 2e-5 * np.abs(table).max(), np.abs(got - want).max()


def pin_rotary_hf_matches_torch(o):
    import torch
    rng = _rng(31)
    T, H, D, rot = 9, 3, 16, 8
    pos = rng.integers(0, 5000, (3, T))
    inv = o.rope_inv_freq(rot, 1e4)
    cos, sin = o.mrope_cos_sin_f32(pos, inv, (2, 1, 1), True)
    for dt, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        x = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32)).to(tdt)
        c = torch.from_numpy(cos).to(tdt)[:, None, :]
        s_ = torch.from_numpy(sin).to(tdt)[:, None, :]
        xr, xp = x[..., :rot], x[..., rot:]
        rh = torch.cat([-xr[..., rot // 2:], xr[..., :rot // 2]], dim=-1)
        want = torch.cat([xr * c + rh * s_, xp], dim=-1).float().numpy().astype(np.float64)
        got = o.apply_rotary_hf(x.float().numpy().astype(np.float64), cos, sin, dt)
        assert (got == want).all(), dt


def pin_hf_rounding_close_to_exact(o):
    # a handful of dtype roundings away from the exact definitions
    rng = _rng(37)
    table = rng.standard_normal((48 * 48, 16)).astype(np.float32).astype(np.float64)
    grids = [(1, 6, 10), (2, 4, 4)]
    exact = o.vis_pos_embed_interpolate(table, grids, 2)
    hf = o.vis_pos_interp_hf(table, grids, 2, "f32")
    assert np.abs(hf - exact).max() <= 1e-5 * (1 + np.abs(exact).max())
    x = rng.standard_normal((5, 2, 12))
    pos = rng.integers(0, 100, (3, 5))
    inv = o.rope_inv_freq(12, 1e4)
    exact = o.mrope_apply(x.astype(np.float32).astype(np.float64), pos, inv, (2, 2, 2), False)
    hf = o.mrope_apply_hf(x.astype(np.float32).astype(np.float64), pos, inv, (2, 2, 2), False, "f32")
    assert np.abs(hf - exact).max() <= 1e-5 * (1 + np.abs(exact).max())


def _interleaved_axis(j, sec):
    """Axis of frequency j in the interleaved layout, from the selection
    rule: H on frequencies 1, 4, 7, ... below 3 s_h, W on 2, 5, 8, ... below
    3 s_w, T on every other one."""
    if j % 3 == 1 and j < 3 * sec[1]:
        return 1
    if j % 3 == 2 and j < 3 * sec[2]:
        return 2
    return 0


def pin_mrope_cos_sin_fp32_angles(o):
    # The interleaved text angles are fp32 products fl32(fl32(pos) * inv_j)
    # of the frequency's own axis; the oracle's cos / sin are the double cos /
    # sin of exactly those angles, and fp32 cos / sin (numpy) agree with them
    # to fp32 rounding.  Selecting axes before or after the cos is the same
    # table (the cos is elementwise).  A position above 2^24 is rounded by
    # the fp32 conversion.
    rng = _rng(53)
    for half, sec, theta in [(64, (24, 20, 20), 5e6), (32, (11, 11, 10), 1e7), (10, (4, 3, 3), 1e4)]:
        L = 40
        pos = rng.integers(0, 300000, (3, L)).astype(np.int64)
        pos[:, 0] = (1 << 24) + 1
        pos[:, 1] = [7, 7, 7]
        inv = o.rope_inv_freq(2 * half, theta)
        cos, sin = o.mrope_cos_sin(pos, inv, sec, True)
        axis = np.array([_interleaved_axis(j, sec) for j in range(half)])
        p32 = pos.astype(np.float32)[axis]                       # [half, L]: the axis each column reads
        ang = (p32 * inv[:, None].astype(np.float32)).T           # [L, half] fp32 products
        ang = np.concatenate([ang, ang], 1).astype(np.float64)
        assert np.abs(np.cos(ang) - cos).max() <= 4e-16 and np.abs(np.sin(ang) - sin).max() <= 4e-16
        c32, s32 = np.cos(ang.astype(np.float32)), np.sin(ang.astype(np.float32))
        assert np.abs(c32 - cos).max() <= 1.2e-7 and np.abs(s32 - sin).max() <= 1.2e-7, (half, sec)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
