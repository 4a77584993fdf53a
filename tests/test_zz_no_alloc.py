"""The allocation-free position-table entry point against the workspace one.

Collected last so that it also runs after every other test in the same
process; it must pass there and alone in a fresh process.  Two calls in a
row on different inputs check that nothing left in the library-owned scratch
by one call changes the next.
"""
import numpy as np
import pytest
import torch

import interpolated_position_encoding_b200 as ipe
from pins import _random_batch

pytestmark = pytest.mark.gpu


def _dev(a, dtype=torch.int32):
    return None if a is None or len(a) == 0 else torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


def _inputs(seed, B):
    types, mask, img, vid = _random_batch(np.random.default_rng([313, seed]), B)
    return _dev(types), _dev(img), _dev(vid), _dev(mask)


def test_static_scratch_matches_workspace_entry_point():
    cases = [_inputs(0, 5), _inputs(1, 3)]
    outs = []
    for ty, img, vid, mask in cases:   # two calls in a row, outputs kept apart
        B, L = ty.shape
        pos = torch.full((3, B, L), -7, dtype=torch.int32, device="cuda")
        deltas = torch.full((B,), -7, dtype=torch.int32, device="cuda")
        ipe.mrope_rope_index_static(ty, img, vid, mask, 2, pos, deltas)
        outs.append((pos, deltas))
    ipe.device_status()
    for (ty, img, vid, mask), (pos, deltas) in zip(cases, outs):
        want_pos, want_deltas = ipe.mrope_rope_index(ty, img, vid, mask, 2)
        ipe.device_status()
        assert torch.equal(pos, want_pos)
        assert torch.equal(deltas, want_deltas)


def test_static_scratch_rejects_sizes_beyond_its_buffer():
    B, L = 64, 1 << 20     # needs more scratch than the library holds
    assert ipe.rope_index_workspace_bytes(B, L) > ipe.ROPE_INDEX_STATIC_BYTES
    ty = torch.zeros(1, 1, dtype=torch.int32, device="cuda").expand(B, L)
    # a [B, L] view without the memory behind it: the binding refuses it on
    # its size alone, before it looks at layout, outputs or contents
    with pytest.raises(ipe.IpeError, match="bytes of scratch") as e:
        ipe.mrope_rope_index_static(ty, None, None, None, 2, None, None)
    assert e.value.status == ipe.IPE_ELIMIT
    # and the C entry point itself, before it reads any pointer
    rc = ipe.lib().ipe_mrope_rope_index_static(None, None, 4, B, L, None, 0, None, 0, 4, 2, None, None, None)
    assert rc == ipe.IPE_ELIMIT
    assert b"bytes of scratch" in ipe.lib().ipe_last_error()
