"""The device entry points inside a captured CUDA graph: replaying the graph
gives the same results as calling them eagerly (after one eager call per
entry point, which creates the library's per-device streams and events
outside the capture)."""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, scale=1.0):
    return torch.from_numpy(wl.normal_bf16(rng, shape, scale).view(np.int16)).view(torch.bfloat16).cuda()


def test_graph_replay_matches_eager():
    rng = np.random.default_rng(21)
    T, hq, hk, D, rot = 512, 8, 2, 128, 64
    q0, k0 = _bf16(rng, (T, hq, D)), _bf16(rng, (T, hk, D))
    pos = torch.from_numpy(rng.integers(0, 20000, (3, T)).astype(np.int32)).cuda()
    inv = ipe.rope_inv_freq(rot, 1e6)
    w = _bf16(rng, (D,), 0.5)
    grid = [(1, 16, 24), (2, 8, 8)]
    N = sum(t * h * ww for t, h, ww in grid)
    table = _bf16(rng, (48 * 48, 1152), 0.02)
    qv0, kv0 = _bf16(rng, (N, 16, 72)), _bf16(rng, (N, 16, 72))
    B = 16
    dq0, dk0 = _bf16(rng, (B, hq, D)), _bf16(rng, (B, hk, D))
    seq = torch.arange(100, 100 + B, dtype=torch.int32, device="cuda")
    # a position table of 3 x 2100 slots: text, an image across a tile edge, text
    types = torch.zeros(3, 2100, dtype=torch.int32, device="cuda")
    types[:, 1000:1096] = 1
    img = torch.tensor([[1, 16, 24]] * 3, dtype=torch.int32, device="cuda")
    ws = torch.empty(ipe.rope_index_workspace_bytes(3, 2100, 3, 0), dtype=torch.uint8, device="cuda")

    def run(q, k, qn, kn, qv, kv, out, dq, dk, pt, dl, stream=None):
        ipe.mrope_apply(q, k, pos, inv, (12, 10, 10), True, stream=stream)
        ipe.qk_norm_mrope(qn, kn, w, w, pos, inv, (12, 10, 10), True, stream=stream)
        ipe.vis_pos_interp_rope2d(table, grid, qv, kv, 2, 1e4, out=out, stream=stream)
        ipe.mrope_decode(dq, dk, seq, inv, stream=stream)
        ipe.mrope_rope_index(types, img, None, None, 2, pt, dl, ws, stream=stream)

    # eager reference (also the first call of each entry point)
    def tables():
        return [torch.full((3, 3, 2100), -1, dtype=torch.int32, device="cuda"),
                torch.full((3,), -1, dtype=torch.int32, device="cuda")]

    ref = [q0.clone(), k0.clone(), q0.clone(), k0.clone(), qv0.clone(), kv0.clone(),
           torch.empty(N, 1152, dtype=torch.bfloat16, device="cuda"), dq0.clone(), dk0.clone()] + tables()
    run(*ref)
    torch.cuda.synchronize()
    ipe.device_status()

    bufs = [q0.clone(), k0.clone(), q0.clone(), k0.clone(), qv0.clone(), kv0.clone(),
            torch.empty(N, 1152, dtype=torch.bfloat16, device="cuda"), dq0.clone(), dk0.clone()] + tables()
    inputs = [q0, k0, q0, k0, qv0, kv0, None, dq0, dk0, None, None]
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            run(*bufs, stream=s)
    for _ in range(2):      # the in-place operands are reset before every replay
        for b, x in zip(bufs, inputs):
            if x is not None:
                b.copy_(x)
        g.replay()
        torch.cuda.synchronize()
        for got, want in zip(bufs, ref):
            assert torch.equal(got, want)
    ipe.device_status()
