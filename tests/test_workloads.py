"""Seeded synthetic inputs: position layout, bf16 cast and workload sizes (CPU only)."""
import numpy as np
import pytest

import workloads as wl
from pins import golden


def test_positions_match_worked_table():
    # t0, S (text), a [1, 4, 6] image with merge 2, E, t1 (text)
    pos, nxt = wl.build_positions([("text", 2), ("vision", (1, 4, 6)), ("text", 2)], merge=2)
    want = {k[0]: [int(v) for v in vals] for k, vals in golden("positions_l10.txt")}
    assert pos.tolist() == [want["T"], want["H"], want["W"]]
    assert nxt == 7


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0, 65504.0], np.float32)
    b = wl.f32_to_bf16_bits(x)
    back = wl.bf16_bits_to_f32(b)
    # ties go to the even mantissa; exactly representable values are unchanged
    assert back.tolist() == [1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5, 0.0, 65536.0]
    r = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    err = np.abs(wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(r)) - r)
    assert (err <= np.abs(r) * 2.0 ** -8).all()


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_workload_layout(name):
    w = wl.WORKLOADS[name]
    if w.text is not None:
        t = w.text
        assert wl.segments_length(t.segments, t.merge) == t.T
        assert sum(t.section) * 2 == t.rot_dim <= t.head_dim
        pos, nxt = wl.build_positions(t.segments, t.merge)
        assert pos.shape == (3, t.T) and pos.dtype == np.int32
        assert pos.min() >= 0 and pos.max() < nxt < 2 ** 24
        # text columns carry equal rows
        same = (pos[0] == pos[1]) & (pos[1] == pos[2])
        assert same.sum() >= t.T // 2
    if w.vision is not None:
        v = w.vision
        assert all(h % v.merge == 0 and ww % v.merge == 0 for _, h, ww in v.grid_thw)


def test_vision_batch_grids_are_seeded():
    w = wl.WORKLOADS["vision_batch8_bf16"]
    assert len(w.vision.grid_thw) == 8
    assert all(g in wl.VISION_GRID_CHOICES for g in w.vision.grid_thw)
    assert wl._vision_batch8_grids() == w.vision.grid_thw


def test_prefill_layout():
    w = wl.WORKLOADS["prefill_t131072_video"]
    assert wl.n_patches(w.vision) == 65536
    pos, _ = wl.build_positions(w.text.segments)
    # 16 video slices of 32 x 32 merged tokens, each at one T
    vis = pos[0] != pos[1]
    assert (pos[1] != pos[2]).sum() > 0
    assert vis.sum() <= 16 * 1024


def test_inputs_reproducible():
    w = wl.WORKLOADS["vision_16x16_f32"]
    a, b = wl.vision_inputs(w), wl.vision_inputs(w)
    assert np.array_equal(a["table"], b["table"]) and a["table"].dtype == np.float32
    assert a["q"].shape == (256, 16, 72)
    assert not np.array_equal(a["q"], a["k"])
    assert abs(float(a["table"].std()) - 0.02) < 1e-3
