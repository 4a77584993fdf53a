"""Position table on the device (through the C ABI) against the oracle.

Integer work: positions and deltas must match the oracle bit for bit.  Inputs
that only the device can detect (a run longer or shorter than its grid, grids
that run out, unknown types) must be reported through the device status word.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from pins import _random_batch

pytestmark = pytest.mark.gpu


def _dev(a, dtype=torch.int32):
    return None if a is None else torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


def run_gpu(types, mask, img, vid, merge=2, dtype=torch.int32, gdtype=torch.int32):
    img = None if img is None or len(img) == 0 else img
    vid = None if vid is None or len(vid) == 0 else vid
    pos, deltas = ipe.mrope_rope_index(_dev(types, dtype), _dev(img, gdtype), _dev(vid, gdtype),
                                       _dev(mask, dtype), merge)
    ipe.device_status()
    return pos.cpu().numpy().astype(np.int64), deltas.cpu().numpy().astype(np.int64)


def check(orc, types, mask, img, vid, merge=2, **kw):
    want, wd = orc.rope_index(types, mask, img, vid, merge)
    got, gd = run_gpu(types, mask, img, vid, merge, **kw)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} coordinates differ, first at {bad[:5].tolist()}"
    assert (gd == wd).all(), (gd[:8], wd[:8])


def test_worked_table(orc):
    types = [[0, 0, 1, 1, 1, 1, 1, 1, 0, 0]]
    pos, deltas = run_gpu(types, None, [[1, 4, 6]], None)
    assert pos[:, 0].tolist() == [[0, 1, 2, 2, 2, 2, 2, 2, 5, 6], [0, 1, 2, 2, 2, 3, 3, 3, 5, 6],
                                  [0, 1, 2, 3, 4, 2, 3, 4, 5, 6]]
    assert deltas.tolist() == [-3]


@pytest.mark.parametrize("seed", range(6))
def test_random_small_batches(orc, seed):
    rng = np.random.default_rng([77, seed])
    types, mask, img, vid = _random_batch(rng, 1 + seed)
    check(orc, types, mask, img, vid)


@pytest.mark.parametrize("ids,grids", [(torch.int64, torch.int64), (torch.int32, torch.int64),
                                       (torch.int64, torch.int32)])
def test_int64_inputs(orc, ids, grids):
    types, mask, img, vid = _random_batch(np.random.default_rng(5), 4)
    check(orc, types, mask, img, vid, dtype=ids, gdtype=grids)


def _long_batch(rng, B, L, pad_max):
    """B sequences of many segments filling about L slots, so runs, padding
    and the open vision run all cross 1024-slot tile boundaries."""
    seqs, img, vid = [], [], []
    for _ in range(B):
        ty = []
        target = L - int(rng.integers(0, pad_max + 1))
        while True:
            seg = [0] * int(rng.integers(1, 40))
            kind = rng.integers(0, 4)
            if kind == 1:
                t, h, w = int(rng.integers(1, 3)), 2 * int(rng.integers(1, 24)), 2 * int(rng.integers(1, 24))
                seg += [1] * (t * (h // 2) * (w // 2))
                g = ("i", [t, h, w])
            elif kind == 2:
                t, h, w = int(rng.integers(1, 4)), 2 * int(rng.integers(1, 20)), 2 * int(rng.integers(1, 20))
                for _ in range(t):
                    seg += [0] * int(rng.integers(1, 3)) + [2] * ((h // 2) * (w // 2))
                g = ("v", [t, h, w])
            else:
                seg += [3] * int(rng.integers(0, 30)) if kind == 3 else []
                g = None
            if len(ty) + len(seg) > target:
                break
            ty += seg
            if g is not None:
                (img if g[0] == "i" else vid).append(g[1])
        seqs.append(ty)
    types = np.zeros((B, L), np.int64)
    mask = np.zeros((B, L), np.int64)
    for b, ty in enumerate(seqs):
        off = int(rng.integers(0, L - len(ty) + 1))
        types[b, off:off + len(ty)] = ty
        mask[b, off:off + len(ty)] = 1
        # padding carrying vision types must not start runs
        types[b, :off] = rng.integers(0, 3, off)
    return types, mask, np.array(img, np.int64).reshape(-1, 3), np.array(vid, np.int64).reshape(-1, 3)


@pytest.mark.parametrize("B,L,pad", [(1, 5000, 0), (3, 9000, 3000), (8, 4100, 1500), (40, 2100, 300)])
def test_multi_tile_batches(orc, B, L, pad):
    types, mask, img, vid = _long_batch(np.random.default_rng([B, L]), B, L, pad)
    check(orc, types, mask, img, vid)
    # the same without a mask: the padding becomes real slots only where it is text
    keep_all = np.where(mask == 1, types, 0)
    check(orc, keep_all, None, img, vid)


def _many_images_batch(rng, B, L):
    """B samples of L slots, each a run of small images (2 x 2 merged slots)
    between single text slots, with a few padded slots at the end."""
    types = np.zeros((B, L), np.int64)
    mask = np.ones((B, L), np.int64)
    img = []
    for b in range(B):
        l = 0
        while l + 6 <= L - 4:
            types[b, l + 1:l + 5] = 1          # text, then a (1, 4, 4) image: 4 slots
            img.append([1, 4, 4])
            l += 5 + int(rng.integers(0, 3))
        mask[b, L - int(rng.integers(0, 4)):] = 0
    return types, mask, np.array(img, np.int64)


def test_carry_scan_over_many_chunks(orc):
    # more than 1024 tiles, with runs, padding and samples crossing tile
    # edges and many look-back windows
    types, mask, img, vid = _long_batch(np.random.default_rng(77), 520, 2100, 400)
    assert 520 * 3 > 1024
    check(orc, types, mask, img, vid)


def test_scan_over_many_waves_of_tiles(orc):
    # more tiles than the GPU holds at once (several waves of blocks): tiles
    # look back across windows whose blocks have finished or not yet
    # started, and samples and runs cross tile edges
    types, mask, img, vid = _long_batch(np.random.default_rng(79), 2100, 3100, 500)
    assert 2100 * 4 > 6000
    check(orc, types, mask, img, vid)


def test_grid_prefix_over_many_chunks(orc):
    # more than 1024 image grids (their prefix sums are scanned 1024 at a time)
    types, mask, img = _many_images_batch(np.random.default_rng(78), 8, 1800)
    assert img.shape[0] > 2048
    check(orc, types, mask, img, None)


def test_masked_slot_inside_a_run(orc):
    # a dropped slot inside an image run does not split it
    types = [[0, 1, 1, 1, 0, 1, 1, 1, 0] + [0] * 1100]
    mask = [[1, 1, 1, 1, 0, 1, 1, 1, 1] + [1] * 1100]
    check(orc, types, mask, [[1, 4, 6]], None)


def test_run_across_tiles_and_long_padding(orc):
    # an image run that starts before a long dropped stretch and ends after it
    L = 5000
    types = np.zeros((2, L), np.int64)
    mask = np.ones((2, L), np.int64)
    types[0, 1000:1010] = 1
    mask[0, 1005:3500] = 0
    types[0, 3500:3507] = 1            # 5 + 7 kept slots: a (1, 6, 8) grid
    types[1, 2040:2060] = 2            # a 20-slot video slice across the tile edge
    check(orc, types, mask, [[1, 6, 8]], [[1, 8, 10]])


def test_edges(orc):
    # L = 0: deltas 0
    pos, deltas = ipe.mrope_rope_index(torch.zeros(3, 0, dtype=torch.int32, device="cuda"))
    ipe.device_status()
    assert pos.shape == (3, 3, 0) and deltas.cpu().tolist() == [0, 0, 0]
    # B = 0: nothing
    pos, deltas = ipe.mrope_rope_index(torch.zeros(0, 7, dtype=torch.int32, device="cuda"))
    assert pos.shape == (3, 0, 7) and deltas.shape == (0,)
    # a sample with every slot dropped
    check(orc, [[0, 1, 1], [0, 0, 0]], [[1, 1, 1], [0, 0, 0]], [[1, 1, 2]], None, merge=1)
    # merge 1 and an image with two frames
    check(orc, [[0] + [1] * 12 + [0] * 3], None, [[2, 2, 3]], None, merge=1)


def _segments_batch(segments, merge):
    """Types and grids of one sample laid out from (kind, arg) segments:
    text and audio slots, and each vision segment as a video slice run."""
    types, vid = [], []
    for kind, arg in segments:
        if kind == "text":
            types += [0] * int(arg)
        elif kind == "audio":
            types += [3] * int(arg)
        else:
            t, h, w = arg
            assert t == 1
            types += [2] * ((h // merge) * (w // merge))
            vid.append([1, h, w])
    return np.array([types], np.int64), np.array(vid, np.int64).reshape(-1, 3)


@pytest.mark.parametrize("name", ["text_t4096_qwen35", "text_t32768_omni", "prefill_t131072_video"])
def test_workload_tables(orc, name):
    t = wl.WORKLOADS[name].text
    types, vid = _segments_batch(t.segments, t.merge)
    check(orc, types, None, None, vid, t.merge)
    # and the positions the rotary benchmarks feed the kernels
    pos, _ = run_gpu(types, None, None, vid, t.merge)
    want, _ = wl.build_positions(t.segments, t.merge)
    assert (pos[:, 0] == want).all()


def test_batched_prefill(orc):
    # 16 copies of the 4096-slot mixed sample, left-padded by varying amounts
    t = wl.WORKLOADS["text_t4096_qwen35"].text
    one, vid1 = _segments_batch(t.segments, t.merge)
    B, L = 16, one.shape[1] + 300
    types = np.zeros((B, L), np.int64)
    mask = np.zeros((B, L), np.int64)
    for b in range(B):
        off = 20 * b
        types[b, off:off + one.shape[1]] = one[0]
        mask[b, off:off + one.shape[1]] = 1
    check(orc, types, mask, None, np.concatenate([vid1] * B), t.merge)


@pytest.mark.parametrize("case,code", [
    ("too_few_grids", 16), ("slices_joined", 17), ("run_too_long", 17), ("bad_type", 18), ("bad_grid", 19)])
def test_device_reports(case, code):
    types = [[0, 1, 1, 1, 1, 1, 1, 0]]
    img = [[1, 4, 6]]
    vid = None
    if case == "too_few_grids":
        types = [[0, 1, 1, 1, 1, 1, 1, 0, 1, 1, 1, 1, 1, 1]]
    elif case == "slices_joined":
        types, img, vid = [[0, 2, 2, 2, 2, 0]], None, [[2, 2, 4]]
    elif case == "run_too_long":
        types = [[0, 1, 1, 1, 1, 1, 1, 1, 0]]
    elif case == "bad_type":
        types = [[0, 7, 0]]
        img = None
    elif case == "bad_grid":
        img = [[0, 4, 6]]
    ipe.mrope_rope_index(_dev(types), _dev(img), _dev(vid), None, 2)
    with pytest.raises(ipe.IpeError) as e:
        ipe.device_status()
    assert e.value.status == ipe.IPE_EDEVICE and f"device fault {code}:" in str(e.value)
    ipe.device_status()   # the word was cleared


def test_host_rejects():
    t = torch.zeros(2, 8, dtype=torch.int32, device="cuda")
    with pytest.raises(ipe.IpeError):
        ipe.mrope_rope_index(t, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ipe.IpeError):
        ipe.mrope_rope_index(t, spatial_merge_size=0)
    with pytest.raises(ValueError):
        ipe.mrope_rope_index(t.float())
