"""The Python binding has no CPU path: every device entry point refuses host
tensors (and host devices) with a TypeError before anything is launched."""
import pytest
import torch

import interpolated_position_encoding_b200 as ipe

BF = torch.bfloat16
T, HQ, HK, D = 8, 2, 1, 128


def _calls():
    q, k = torch.zeros(T, HQ, D, dtype=BF), torch.zeros(T, HK, D, dtype=BF)
    pos = torch.zeros(3, T, dtype=torch.int32)
    inv = ipe.rope_inv_freq(64, 1e4)
    w = torch.zeros(D, dtype=BF)
    cs = torch.zeros(T, 64)
    table = torch.zeros(48 * 48, 64, dtype=BF)
    qv, kv = torch.zeros(16, 2, 72, dtype=BF), torch.zeros(16, 2, 72, dtype=BF)
    sec = (11, 11, 10)
    return {
        "mrope_apply": lambda: ipe.mrope_apply(q, k, pos, inv, sec),
        "mrope_apply hf": lambda: ipe.mrope_apply(q, k, pos, inv, sec, rounding="hf"),
        "apply_rotary_partial": lambda: ipe.apply_rotary_partial(q, k, cs, cs),
        "apply_rotary_partial hf": lambda: ipe.apply_rotary_partial(q, k, cs, cs, rounding="hf"),
        "mrope_cos_sin": lambda: ipe.mrope_cos_sin(pos, inv, sec),
        "qk_norm_mrope": lambda: ipe.qk_norm_mrope(q, k, w, w, pos, inv, sec),
        "mrope_decode": lambda: ipe.mrope_decode(q, k, torch.zeros(T, dtype=torch.int32), inv),
        "mrope_rope_index": lambda: ipe.mrope_rope_index(torch.zeros(1, 16, dtype=torch.int32)),
        "mrope_rope_index_static": lambda: ipe.mrope_rope_index_static(
            torch.zeros(1, 16, dtype=torch.int32), None, None, None, 2, torch.zeros(3, 1, 16, dtype=torch.int32),
            torch.zeros(1, dtype=torch.int32)),
        "vis_pos_interp": lambda: ipe.vis_pos_interp(table, [(1, 4, 4)]),
        "vis_pos_interp hf": lambda: ipe.vis_pos_interp(table, [(1, 4, 4)], rounding="hf"),
        "vis_rope2d": lambda: ipe.vis_rope2d(qv, kv, [(1, 4, 4)]),
        "vis_pos_interp_rope2d": lambda: ipe.vis_pos_interp_rope2d(table, [(1, 4, 4)], qv, kv),
        "mrope_axis_map": lambda: ipe.mrope_axis_map(32, sec, device="cpu"),
        "vis_interp_plan": lambda: ipe.vis_interp_plan([(1, 4, 4)], device="cpu"),
    }


@pytest.mark.parametrize("name", sorted(_calls()))
def test_host_tensors_are_refused(name):
    with pytest.raises(TypeError, match="CUDA"):
        _calls()[name]()


def test_unknown_rounding_is_refused():
    with pytest.raises(ValueError):
        ipe._rounding("bf16")


def test_static_scratch_size_refused_before_any_device_work():
    # sizes whose scratch exceeds the library's fixed buffer are refused on
    # the sizes alone, whatever the tensors are
    B, L = 64, 1 << 20
    ty = torch.zeros(1, 1, dtype=torch.int32).expand(B, L)
    with pytest.raises(ipe.IpeError, match="bytes of scratch") as e:
        ipe.mrope_rope_index_static(ty, None, None, None, 2, None, None)
    assert e.value.status == ipe.IPE_ELIMIT
