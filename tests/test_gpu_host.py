"""Host-buffer entry points: chunked, overlapped copies around the same
kernels must give exactly the device entry points' results, also when the
staging buffers are reused by the next call before the previous call's
copies back have finished."""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, scale=1.0):
    return torch.from_numpy(wl.normal_bf16(rng, shape, scale).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("T,chunk", [(5000, 1024), (4096, 4096), (333, 100)])
def test_mrope_apply_host_matches_device(T, chunk):
    rng = np.random.default_rng([T, chunk])
    hq, hk, D, rot = 6, 2, 128, 64
    inv = ipe.rope_inv_freq(rot, 1e6)
    q_dev = torch.empty(T, hq, D, dtype=torch.bfloat16, device="cuda")
    k_dev = torch.empty(T, hk, D, dtype=torch.bfloat16, device="cuda")
    p_dev = torch.empty(3, T, dtype=torch.int32, device="cuda")
    results = []
    for call in range(2):      # two calls in a row on the same staging buffers
        q, k = _bf16(rng, (T, hq, D)).pin_memory(), _bf16(rng, (T, hk, D)).pin_memory()
        pos = torch.from_numpy(rng.integers(0, 50000, (3, T)).astype(np.int32)).pin_memory()
        want_q, want_k = q.cuda(), k.cuda()
        ipe.mrope_apply(want_q, want_k, pos.cuda(), inv, (12, 10, 10), True)
        q_out, k_out = torch.empty_like(q).pin_memory(), torch.empty_like(k).pin_memory()
        ipe.mrope_apply_host(q, k, pos, inv, (12, 10, 10), True, q_dev, k_dev, p_dev, q_out, k_out,
                             chunk_tokens=chunk, join=(call == 1))
        results.append((q_out, k_out, want_q, want_k))
    ipe.host_join()
    torch.cuda.synchronize()
    ipe.device_status()
    for q_out, k_out, want_q, want_k in results:
        assert torch.equal(q_out, want_q.cpu()) and torch.equal(k_out, want_k.cpu())


@pytest.mark.parametrize("rot", [64, 128])
def test_mrope_apply_host_in_place(rot):
    # in place only the rotary slices cross the link; the rest stays as it was
    rng = np.random.default_rng([rot, 9])
    T, hq, hk, D = 3000, 4, 2, 128
    inv = ipe.rope_inv_freq(rot, 1e6)
    sec = (rot // 2 - 2 * (rot // 6), rot // 6, rot // 6)
    q, k = _bf16(rng, (T, hq, D)).pin_memory(), _bf16(rng, (T, hk, D)).pin_memory()
    pos = torch.from_numpy(rng.integers(0, 50000, (3, T)).astype(np.int32)).pin_memory()
    want_q, want_k = q.cuda(), k.cuda()
    ipe.mrope_apply(want_q, want_k, pos.cuda(), inv, sec, True)
    q_dev, k_dev = torch.empty_like(want_q), torch.empty_like(want_k)
    p_dev = torch.empty(3, T, dtype=torch.int32, device="cuda")
    ipe.mrope_apply_host(q, k, pos, inv, sec, True, q_dev, k_dev, p_dev, chunk_tokens=1000)
    torch.cuda.synchronize()
    ipe.device_status()
    assert torch.equal(q, want_q.cpu()) and torch.equal(k, want_k.cpu())


def test_vis_rope2d_host_groups_and_splits():
    # small images grouped into chunks, a video split into frame ranges
    grid = [(1, 16, 16), (1, 8, 12), (6, 16, 20), (1, 4, 4), (2, 10, 10)]
    N = sum(t * h * w for t, h, w in grid)
    rng = np.random.default_rng(4)
    q, k = _bf16(rng, (N, 16, 72)).pin_memory(), _bf16(rng, (N, 16, 72)).pin_memory()
    want_q, want_k = q.cuda(), k.cuda()
    ipe.vis_rope2d(want_q, want_k, grid, 2, 1e4)
    q_dev, k_dev = torch.empty_like(want_q), torch.empty_like(want_k)
    qo, ko = torch.empty_like(q).pin_memory(), torch.empty_like(k).pin_memory()
    ipe.vis_rope2d_host(q, k, grid, q_dev, k_dev, 2, 1e4, qo, ko, chunk_rows=700)
    torch.cuda.synchronize()
    ipe.device_status()
    assert torch.equal(qo, want_q.cpu()) and torch.equal(ko, want_k.cpu())


def test_vis_pos_interp_host_and_pageable_memory():
    grid = [(3, 32, 32), (1, 48, 64), (1, 8, 8)]
    N = sum(t * h * w for t, h, w in grid)
    rng = np.random.default_rng(6)
    table = _bf16(rng, (48 * 48, 1152), 0.02)               # pageable
    want = ipe.vis_pos_interp(table.cuda(), grid, 2)
    out = torch.empty(N, 1152, dtype=torch.bfloat16)        # pageable
    t_dev, o_dev = torch.empty_like(table, device="cuda"), torch.empty_like(want)
    ipe.vis_pos_interp_host(table, grid, out, t_dev, o_dev, 2, chunk_rows=1500)
    torch.cuda.synchronize()
    ipe.device_status()
    assert torch.equal(out, want.cpu())


def test_host_entry_points_reject_device_tensors():
    q = torch.zeros(4, 1, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        ipe.mrope_apply_host(q, q, torch.zeros(3, 4, dtype=torch.int32), ipe.rope_inv_freq(64, 1e4), (12, 10, 10),
                             True, q, q, torch.zeros(3, 4, dtype=torch.int32, device="cuda"))
