"""Canary guards around every output: no kernel writes outside its tensors.

Each entry point writes through a view in the middle of a larger buffer
whose bytes all start as 0xA5; after the call (and the device status
check) the bytes before and after the view must be untouched, and the view
itself must have been written.  The values are checked against the oracle
elsewhere; this file checks only where the kernels write.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import bf16_to_gpu

pytestmark = pytest.mark.gpu

PAD = 3          # guard rows on each side, at least
SENTINEL = 0xA5


def guarded(shape, dtype):
    """(buffer, view, pad): the view is rows pad .. pad + shape[0] of the
    buffer, pad >= PAD rows chosen so that the view starts 16-byte aligned
    (as an allocation would)."""
    n = shape[0]
    row_bytes = int(np.prod(shape[1:], dtype=np.int64)) * torch.tensor([], dtype=dtype).element_size()
    pad = PAD
    while (pad * row_bytes) % 16:
        pad += 1
    big = torch.empty((n + 2 * pad,) + tuple(shape[1:]), dtype=dtype, device="cuda")
    big.view(-1).view(torch.uint8).fill_(SENTINEL)
    return big, big[pad:pad + n], pad


def assert_guards(big, pad, what):
    torch.cuda.synchronize()
    n = big.shape[0] - 2 * pad
    flat = big.reshape(big.shape[0], -1).view(torch.uint8)
    assert bool((flat[:pad] == SENTINEL).all()), f"{what}: a write before the output"
    assert bool((flat[pad + n:] == SENTINEL).all()), f"{what}: a write after the output"
    assert not bool((flat[pad:pad + n] == SENTINEL).all()), f"{what}: nothing written"


def _vision(dtype):
    rng = np.random.default_rng(21)
    G, C, heads, hd = 48, 1152, 16, 72
    grid = [(2, 8, 12), (1, 16, 16)]
    N = sum(t * h * w for t, h, w in grid)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    conv = bf16_to_gpu if dtype == "bf16" else (lambda a: torch.from_numpy(a).cuda())
    table = conv(gen(rng, (G * G, C), 0.02))
    q, k = conv(gen(rng, (N, heads, hd))), conv(gen(rng, (N, heads, hd)))
    return grid, N, table, q, k, tdt


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rounding", ["fp32", "hf"])
def test_interpolation_writes_only_its_output(dtype, rounding):
    grid, N, table, _, _, tdt = _vision(dtype)
    big, out, pad = guarded((N, table.shape[1]), tdt)
    ipe.vis_pos_interp(table, grid, 2, out=out, rounding=rounding)
    ipe.device_status()
    assert_guards(big, pad, f"vis_pos_interp {dtype} {rounding}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_vision_rotary_and_one_call_write_only_their_rows(dtype):
    grid, N, table, q, k, tdt = _vision(dtype)
    bq, gq, pq = guarded(tuple(q.shape), tdt)
    bk, gk, pk = guarded(tuple(k.shape), tdt)
    gq.copy_(q)
    gk.copy_(k)
    ipe.vis_rope2d(gq, gk, grid, 2, 1e4)
    ipe.device_status()
    assert_guards(bq, pq, f"vis_rope2d q {dtype}")
    assert_guards(bk, pk, f"vis_rope2d k {dtype}")
    bo, out, po = guarded((N, table.shape[1]), tdt)
    ipe.vis_pos_interp_rope2d(table, grid, gq, gk, 2, 1e4, out=out)
    ipe.device_status()
    for b, p, nm in ((bo, po, "out"), (bq, pq, "q"), (bk, pk, "k")):
        assert_guards(b, p, f"vis_pos_interp_rope2d {nm} {dtype}")


def _text(T=301, hq=24, hk=4, D=256, rot=64):
    rng = np.random.default_rng([22, T])
    q = bf16_to_gpu(wl.normal_bf16(rng, (T, hq, D)))
    k = bf16_to_gpu(wl.normal_bf16(rng, (T, hk, D)))
    pos = torch.from_numpy(rng.integers(0, 50000, (3, T)).astype(np.int32)).cuda()
    return q, k, pos, ipe.rope_inv_freq(rot, 1e7)


def test_cos_sin_tables_write_only_their_rows():
    _, _, pos, inv = _text()
    T = pos.shape[1]
    bc, cos, pc = guarded((T, 2 * inv.numel()), torch.float32)
    bs, sin, ps = guarded((T, 2 * inv.numel()), torch.float32)
    ipe.mrope_cos_sin(pos, inv, (11, 11, 10), True, cos, sin)
    ipe.device_status()
    assert_guards(bc, pc, "mrope_cos_sin cos")
    assert_guards(bs, ps, "mrope_cos_sin sin")


@pytest.mark.parametrize("path", ["mrope_apply", "mrope_apply_hf", "apply_rotary_partial", "qk_norm_mrope"])
@pytest.mark.parametrize("shape", [(301, 24, 4, 256, 64), (77, 32, 4, 128, 128)], ids=["rot64_of_256", "rot128_whole"])
def test_text_rotations_write_only_their_rows(path, shape):
    T, hq, hk, D, rot = shape
    q, k, pos, inv = _text(T, hq, hk, D, rot)
    section = (11, 11, 10) if rot == 64 else (24, 20, 20)
    bq, gq, pq = guarded(tuple(q.shape), torch.bfloat16)
    bk, gk, pk = guarded(tuple(k.shape), torch.bfloat16)
    gq.copy_(q)
    gk.copy_(k)
    if path == "mrope_apply":
        ipe.mrope_apply(gq, gk, pos, inv, section, True)
    elif path == "mrope_apply_hf":
        ipe.mrope_apply(gq, gk, pos, inv, section, True, rounding="hf")
    elif path == "apply_rotary_partial":
        cos, sin = ipe.mrope_cos_sin(pos, inv, section, True)
        ipe.apply_rotary_partial(gq, gk, cos, sin)
    else:
        w = torch.ones(D, dtype=torch.bfloat16, device="cuda")
        ipe.qk_norm_mrope(gq, gk, w, w, pos, inv, section, True)
    ipe.device_status()
    assert_guards(bq, pq, f"{path} q {shape}")
    assert_guards(bk, pk, f"{path} k {shape}")


def test_position_table_writes_only_its_outputs():
    L = 3 * 1024 + 17
    types = torch.zeros(1, L, dtype=torch.int32, device="cuda")
    types[0, 1500:1524] = 1                         # a (1, 8, 12) image, merged 2 x 2
    img = torch.tensor([[1, 8, 12]], dtype=torch.int32, device="cuda")
    bp, pflat, pp = guarded((3 * L,), torch.int32)
    bd, deltas, pd = guarded((1,), torch.int32)
    ipe.mrope_rope_index(types, img, None, None, 2, pflat.view(3, 1, L), deltas)
    ipe.device_status()
    assert_guards(bp, pp, "mrope_rope_index position_ids")
    assert_guards(bd, pd, "mrope_rope_index rope_deltas")
