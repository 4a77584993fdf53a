"""Failure path of the kernels that wait: a bounded wait that runs out.

The test hook makes the producer of a TMA-fed kernel skip one tile's loads
(or one tile of the position-table scan publish nothing), so the warps
waiting for it give up after a short limit, record a fault in the device
status word and return.  Nothing faults or hangs: the host reads the
status, the context stays usable, and the next launch is correct.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import bf16_to_gpu

pytestmark = pytest.mark.gpu

SHORT_WAIT = 1 << 24      # SM cycles, about 9 ms


def _text_case(T=4096):
    rng = np.random.default_rng([5, T])
    pos = torch.from_numpy(np.tile(np.arange(T, dtype=np.int32), (3, 1))).cuda()
    q = bf16_to_gpu(wl.normal_bf16(rng, (T, 24, 256)))
    k = bf16_to_gpu(wl.normal_bf16(rng, (T, 4, 256)))
    return pos, q, k


def test_status_is_clean_after_normal_launches():
    pos, q, k = _text_case()
    ipe.mrope_apply(q, k, pos, ipe.rope_inv_freq(64, 1e7), (11, 11, 10))
    ipe.device_status()


@pytest.mark.parametrize("path", ["mrope_apply", "vis_rope2d", "apply_rotary_partial", "mrope_apply_wide"])
def test_skipped_tile_times_out_and_recovers(path):
    # the first three take a ring of three or more stages (a stage freed one
    # row late); the wide rows (9 KB: 36 heads of 128 channels, rotated
    # whole) take two stages at one block per SM (a stage freed at once)
    inv = ipe.rope_inv_freq(64, 1e7)
    pos, q, k = _text_case()
    if path == "mrope_apply_wide":
        rng = np.random.default_rng([6, 2048])
        pos = torch.from_numpy(np.tile(np.arange(2048, dtype=np.int32), (3, 1))).cuda()
        q = bf16_to_gpu(wl.normal_bf16(rng, (2048, 32, 128)))
        k = bf16_to_gpu(wl.normal_bf16(rng, (2048, 4, 128)))
        inv = ipe.rope_inv_freq(128, 1e6)
    grid = [(4, 16, 32)]
    rng = np.random.default_rng(11)
    vq = bf16_to_gpu(wl.normal_bf16(rng, (2048, 16, 72)))
    vk = bf16_to_gpu(wl.normal_bf16(rng, (2048, 16, 72)))
    cos, sin = ipe.mrope_cos_sin(pos, inv, (11, 11, 10)) if path == "apply_rotary_partial" else (None, None)

    def run(a, b):
        if path == "mrope_apply":
            ipe.mrope_apply(a, b, pos, inv, (11, 11, 10))
        elif path == "mrope_apply_wide":
            ipe.mrope_apply(a, b, pos, inv, (24, 20, 20))
        elif path == "apply_rotary_partial":
            ipe.apply_rotary_partial(a, b, cos, sin)
        else:
            ipe.vis_rope2d(a, b, grid, 2, 1e4)

    a0, b0 = (q, k) if path != "vis_rope2d" else (vq, vk)
    ref_a, ref_b = a0.clone(), b0.clone()
    run(ref_a, ref_b)
    ipe.device_status()

    ipe.debug_inject(3, SHORT_WAIT)
    try:
        bad_a, bad_b = a0.clone(), b0.clone()
        run(bad_a, bad_b)
        with pytest.raises(ipe.IpeError) as err:
            ipe.device_status()
        assert err.value.status == ipe.IPE_EDEVICE
        assert "gave up" in str(err.value)
    finally:
        ipe.debug_inject(-1, 0)
    # the word was cleared, the context works and results are right again
    ipe.device_status()
    good_a, good_b = a0.clone(), b0.clone()
    run(good_a, good_b)
    ipe.device_status()
    assert torch.equal(good_a, ref_a) and torch.equal(good_b, ref_b)
    assert not torch.equal(bad_a, ref_a) or not torch.equal(bad_b, ref_b)


def test_position_table_look_back_times_out_and_recovers():
    # the position-table scan: tile 1 publishes nothing, so the tiles after it
    # give up their look-back, report code 23 and mark themselves failed
    L = 3 * 1024 + 17
    types = torch.zeros(1, L, dtype=torch.int32, device="cuda")
    types[0, 1500:1524] = 1                         # a (1, 8, 12) image across tiles 1 and 2
    img = torch.tensor([[1, 8, 12]], dtype=torch.int32, device="cuda")
    ref_pos, ref_d = ipe.mrope_rope_index(types, img, None, None, 2)
    ipe.device_status()
    ipe.debug_inject(1, SHORT_WAIT)
    try:
        ipe.mrope_rope_index(types, img, None, None, 2)
        with pytest.raises(ipe.IpeError) as err:
            ipe.device_status()
        assert err.value.status == ipe.IPE_EDEVICE and "device fault 23:" in str(err.value)
    finally:
        ipe.debug_inject(-1, 0)
    ipe.device_status()
    pos, d = ipe.mrope_rope_index(types, img, None, None, 2)
    ipe.device_status()
    assert torch.equal(pos, ref_pos) and torch.equal(d, ref_d)
