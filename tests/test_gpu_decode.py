"""Decode step (through the C ABI) against the oracle.

Positions come from the oracle's decode rule (sequence index plus the rope
delta of a prefill the oracle laid out), the rotation and the optional norm
from the oracle's prefill functions at those positions; the cache rows must be
bit-identical copies of the rotated k rows and of v, and no other slot may
change.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
import workloads as wl
from gpu_helpers import check, gpu_to_f64, host_f64, to_gpu
from pins import _random_batch
from test_gpu_qknorm import check_qk

pytestmark = pytest.mark.gpu


def _prefill_state(orc, B, seed):
    """Sequence indices and deltas of the token after a random prefill."""
    types, mask, img, vid = _random_batch(np.random.default_rng([55, seed]), B)
    _, deltas = orc.rope_index(types, mask, img, vid, 2)
    grown = np.concatenate([mask, np.ones((B, 1), np.int64)], axis=1)
    pos = orc.decode_positions(1, mask=grown, deltas=deltas)[:, :, 0]     # [3, B]
    seq_pos = mask.sum(1)        # cumsum(mask)[-1] - 1 with the new token kept
    return seq_pos.astype(np.int32), deltas.astype(np.int32), pos


def _section(half):
    a = half // 3
    return (half - 2 * a, a, a)


CASES = [  # (B, hq, hk, D, rot, dtype)
    (13, 4, 2, 256, 64, "bf16"),
    (64, 24, 4, 256, 64, "bf16"),     # Qwen3.5 heads
    (9, 8, 4, 128, 128, "bf16"),      # full-dim rotary
    (11, 3, 1, 64, 32, "f32"),
    (5, 2, 2, 128, 128, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_h%d_%d_D%d_r%d_%s" % c)
@pytest.mark.parametrize("norm", [False, True], ids=["rope", "norm_rope"])
@pytest.mark.parametrize("cache", [False, True], ids=["nocache", "cache"])
def test_decode_step(case, norm, cache, orc):
    B, hq, hk, D, rot, dtype = case
    rng = np.random.default_rng([B, hq, D, rot, norm, cache])
    gen = wl.normal_bf16 if dtype == "bf16" else wl.normal_f32
    q, k, v = gen(rng, (B, hq, D), 2.0), gen(rng, (B, hk, D), 2.0), gen(rng, (B, hk, D), 1.0)
    wq, wk = gen(rng, (D,), 0.5), gen(rng, (D,), 0.5)
    seq_pos, deltas, pos = _prefill_state(orc, B, B + D)
    inv = ipe.rope_inv_freq(rot, 1e7)
    oinv = orc.rope_inv_freq(rot, 1e7)
    gq, gk, gv = to_gpu(q, dtype), to_gpu(k, dtype), to_gpu(v, dtype)
    kw = {}
    if norm:
        kw.update(q_weight=to_gpu(wq, dtype), k_weight=to_gpu(wk, dtype), eps=1e-6)
    slots = None
    if cache:
        n_slots = 3 * B + 5
        kc = torch.full((n_slots, hk, D), 7.0, dtype=gq.dtype, device="cuda")
        vc = torch.full((n_slots, hk, D), -3.0, dtype=gq.dtype, device="cuda")
        slots = rng.permutation(n_slots)[:B].astype(np.int64)
        slots[::4] = -1                                      # padding rows: no write
        kw.update(v=gv, k_cache=kc, v_cache=vc, slot_mapping=torch.from_numpy(slots).cuda())
    ipe.mrope_decode(gq, gk, torch.from_numpy(seq_pos).cuda(), inv, torch.from_numpy(deltas).cuda(), **kw)
    ipe.device_status()
    half = rot // 2
    for nm, x, w, g in (("q", q, wq, gq), ("k", k, wk, gk)):
        xf = host_f64(x, dtype)
        what = f"{case} {nm} norm={norm}"
        if norm:
            check_qk(gpu_to_f64(g), xf, host_f64(w, dtype), 1e-6, dtype, pos, oinv, _section(half), True, orc, what)
        else:
            ref, mag = orc.mrope_apply(xf, pos, oinv, _section(half), True, with_mag=True)
            check(gpu_to_f64(g)[..., :rot], ref[..., :rot], mag, dtype, what)
            assert (gpu_to_f64(g)[..., rot:] == xf[..., rot:]).all(), f"{what}: pass-through changed"
    if cache:
        kcn, vcn, gkn, gvn = (t.float().cpu().numpy() for t in (kc, vc, gk, gv))
        written = slots[slots >= 0]
        for b in range(B):
            if slots[b] >= 0:
                assert (kcn[slots[b]] == gkn[b]).all(), f"k_cache slot of token {b}"
                assert (vcn[slots[b]] == gvn[b]).all(), f"v_cache slot of token {b}"
        rest = np.setdiff1d(np.arange(kcn.shape[0]), written)
        assert (kcn[rest] == 7.0).all() and (vcn[rest] == -3.0).all(), "a slot outside slot_mapping changed"
        assert (gvn == host_f64(v, dtype)).all(), "v was modified"


def test_decode_positions_without_deltas(orc):
    # no deltas: the position is the sequence index itself (text-only prompts)
    B, hq, hk, D, rot = 7, 2, 1, 128, 64
    rng = np.random.default_rng(8)
    q, k = wl.normal_bf16(rng, (B, hq, D), 1.0), wl.normal_bf16(rng, (B, hk, D), 1.0)
    seq = np.array([0, 1, 5, 100, 4095, 70000, 16777215], np.int32)
    gq, gk = to_gpu(q, "bf16"), to_gpu(k, "bf16")
    ipe.mrope_decode(gq, gk, torch.from_numpy(seq).cuda(), ipe.rope_inv_freq(rot, 1e6))
    ipe.device_status()
    pos = orc.decode_positions(1, cache_len=seq.astype(np.int64))[:, :, 0]
    ref, mag = orc.mrope_apply(host_f64(q, "bf16"), pos, orc.rope_inv_freq(rot, 1e6), (12, 10, 10), False,
                               with_mag=True)
    check(gpu_to_f64(gq)[..., :rot], ref[..., :rot], mag, "bf16", "q")


def test_decode_matches_prefill_kernel(orc):
    # the decode kernel and the prefill kernel give bit-identical rows for the
    # same positions (same fp32 angles, same arithmetic)
    B, hq, hk, D, rot = 32, 24, 4, 256, 64
    rng = np.random.default_rng(9)
    q, k = wl.normal_bf16(rng, (B, hq, D), 2.0), wl.normal_bf16(rng, (B, hk, D), 2.0)
    wq, wk = wl.normal_bf16(rng, (D,), 0.5), wl.normal_bf16(rng, (D,), 0.5)
    seq = rng.integers(0, 1 << 20, B).astype(np.int32)
    inv = ipe.rope_inv_freq(rot, 1e7)
    a = [to_gpu(q, "bf16"), to_gpu(k, "bf16")]
    b = [to_gpu(q, "bf16"), to_gpu(k, "bf16")]
    gw = (to_gpu(wq, "bf16"), to_gpu(wk, "bf16"))
    ipe.mrope_decode(a[0], a[1], torch.from_numpy(seq).cuda(), inv, q_weight=gw[0], k_weight=gw[1])
    positions = torch.from_numpy(np.stack([seq] * 3)).cuda()
    ipe.qk_norm_mrope(b[0], b[1], gw[0], gw[1], positions, inv, (11, 11, 10), True)
    ipe.device_status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("case,code", [("position", 21), ("slot", 22)])
def test_decode_device_reports(case, code):
    B, D = 4, 128
    q = torch.zeros(B, 2, D, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(B, 1, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(8, 1, D, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([0, 1, 2, 3], dtype=torch.int32, device="cuda")
    slots = torch.tensor([0, 1, 2, 3], dtype=torch.int64, device="cuda")
    if case == "position":
        seq[2] = 1 << 24
    else:
        slots[3] = 8
    ipe.mrope_decode(q, k, seq, ipe.rope_inv_freq(64, 1e6), k_cache=kc, slot_mapping=slots)
    with pytest.raises(ipe.IpeError) as e:
        ipe.device_status()
    assert e.value.status == ipe.IPE_EDEVICE and f"device fault {code}:" in str(e.value)
    ipe.device_status()


def test_decode_host_rejects():
    q = torch.zeros(4, 2, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 1, 128, dtype=torch.bfloat16, device="cuda")
    seq = torch.zeros(4, dtype=torch.int32, device="cuda")
    inv = ipe.rope_inv_freq(64, 1e6)
    with pytest.raises(ipe.IpeError):      # one weight only
        ipe.mrope_decode(q, k, seq, inv, q_weight=torch.ones(128, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ipe.IpeError):      # a cache without slots
        ipe.mrope_decode(q, k, seq, inv, k_cache=torch.zeros(4, 1, 128, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ipe.IpeError):      # head_dim not a power-of-two count of 16-byte chunks
        ipe.mrope_decode(torch.zeros(4, 2, 96, dtype=torch.bfloat16, device="cuda"),
                         torch.zeros(4, 1, 96, dtype=torch.bfloat16, device="cuda"), seq, ipe.rope_inv_freq(32, 1e6))
