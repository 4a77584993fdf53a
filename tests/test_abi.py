"""C ABI of libipe.so without a GPU: exports, host-only entry points and the
argument checks that run before any CUDA call."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import interpolated_position_encoding_b200 as ipe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ipe.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ipe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding():
    assert header_functions() == sorted(ipe.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ipe.lib()._name)
    for name in header_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", ipe.lib()._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ipe_[a-z0-9_]+)$", out, flags=re.M))
    assert set(header_functions()) <= exported


def test_library_is_sm100a_only():
    # The fatbinary holds sm_100a code (and no PTX for other targets).
    out = subprocess.run(["cuobjdump", "--list-elf", ipe.lib()._name], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    arches = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert arches == {"100a"}, arches


def test_version():
    assert ipe.lib().ipe_version() >= 100


@pytest.mark.parametrize("rot,theta", [(64, 1e7), (128, 1e6), (36, 1e4), (8, 1e4), (6, 100.0), (2, 10.0)])
def test_inv_freq_matches_oracle_bitwise(rot, theta, orc):
    got = ipe.rope_inv_freq(rot, theta).numpy()
    want = orc.rope_inv_freq(rot, theta)
    assert got.dtype == np.float32 and np.array_equal(got.view(np.uint32), want.view(np.uint32))


def _err(rc, status):
    assert rc == status, (rc, ipe.lib().ipe_last_error())
    assert ipe.lib().ipe_last_error()


L = ipe.lib()
F = ctypes.c_float
I32 = ctypes.c_int32


def sec(a, b, c):
    return (I32 * 3)(a, b, c)


def inv(n):
    return (F * n)(*([1.0] * n))


FAKE = ctypes.c_void_p(0x1000)     # never dereferenced: every case fails earlier


def test_inv_freq_rejects():
    out = (F * 8)()
    _err(L.ipe_rope_inv_freq(7, 1e4, out), ipe.IPE_EINVAL)
    _err(L.ipe_rope_inv_freq(0, 1e4, out), ipe.IPE_EINVAL)
    _err(L.ipe_rope_inv_freq(8, -1.0, out), ipe.IPE_EINVAL)
    _err(L.ipe_rope_inv_freq(8, float("inf"), out), ipe.IPE_EINVAL)
    _err(L.ipe_rope_inv_freq(1024, 1e4, (F * 512)()), ipe.IPE_ELIMIT)
    _err(L.ipe_rope_inv_freq(8, 1e4, None), ipe.IPE_EINVAL)


def test_mrope_rejects_bad_sections_and_dims():
    # section sums to 31, not 32
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                           sec(11, 10, 10), 1, None), ipe.IPE_EINVAL)
    # negative count
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                           sec(33, -1, 0), 1, None), ipe.IPE_EINVAL)
    # odd rot_dim, rot_dim > head_dim
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 63,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 2, 2, 32, 64, 64, FAKE, inv(32), 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    # unknown dtype, negative T, rot/2 above the limit
    _err(L.ipe_mrope_apply(FAKE, FAKE, 7, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, -1, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 1, 1, 1024, 1024, 1024, FAKE, inv(512), 1024,
                           sec(512, 0, 0), 1, None), ipe.IPE_ELIMIT)
    # q stride smaller than a row
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 100, 1024, FAKE, inv(32), 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    # heads but no pointer
    _err(L.ipe_mrope_apply(None, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)
    # non-finite inverse frequency
    bad = inv(32)
    bad[3] = float("nan")
    _err(L.ipe_mrope_apply(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, bad, 64,
                           sec(11, 11, 10), 1, None), ipe.IPE_EINVAL)


def test_cos_sin_and_axis_map_reject():
    _err(L.ipe_mrope_cos_sin(FAKE, 8, inv(10), 10, sec(4, 3, 2), 1, FAKE, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_cos_sin(FAKE, 8, inv(10), 0, sec(0, 0, 0), 1, FAKE, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_cos_sin(FAKE, 8, inv(10), 10, None, 1, FAKE, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_axis_map(10, sec(4, 3, 4), 1, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_axis_map(300, sec(300, 0, 0), 1, FAKE, None), ipe.IPE_ELIMIT)


def test_apply_rotary_rejects():
    _err(L.ipe_apply_rotary_partial(FAKE, FAKE, ipe.IPE_BF16, 8, 2, 2, 16, 32, 32, FAKE, FAKE, 18, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_apply_rotary_partial(FAKE, FAKE, ipe.IPE_BF16, 8, 2, 2, 16, 32, 32, FAKE, FAKE, 5, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_apply_rotary_partial(FAKE, FAKE, 3, 8, 2, 2, 16, 32, 32, FAKE, FAKE, 8, None), ipe.IPE_EINVAL)
    # element misaligned bf16 pointer
    _err(L.ipe_apply_rotary_partial(ctypes.c_void_p(0x1001), None, ipe.IPE_BF16, 8, 2, 0, 16, 32, 0, FAKE, FAKE,
                                    8, None), ipe.IPE_EALIGN)


def grid(*rows):
    flat = [v for r in rows for v in r]
    return (I32 * len(flat))(*flat), len(rows)


def test_vision_rejects():
    g, n = grid((1, 15, 16))    # h not a multiple of merge
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, None), ipe.IPE_EINVAL)
    g, n = grid((0, 16, 16))
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, None), ipe.IPE_EINVAL)
    g, n = grid((1, 16, 16))
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 48, 1150, g, n, 2, FAKE, None), ipe.IPE_EINVAL)   # hidden % 4
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 0, 1152, g, n, 2, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 48, 1152, g, n, 0, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp(ctypes.c_void_p(0x1002), ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, None),
         ipe.IPE_EALIGN)
    many = (I32 * (3 * 1025))(*([1, 2, 2] * 1025))
    _err(L.ipe_vis_pos_interp(FAKE, ipe.IPE_BF16, 48, 1152, many, 1025, 2, FAKE, None), ipe.IPE_ELIMIT)
    # rope: n_patch mismatch, head_dim not a multiple of 4, theta <= 0
    _err(L.ipe_vis_rope2d(FAKE, FAKE, ipe.IPE_BF16, 255, 16, 72, 1152, 1152, g, n, 2, 1e4, None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_rope2d(FAKE, FAKE, ipe.IPE_BF16, 256, 16, 70, 1120, 1120, g, n, 2, 1e4, None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_rope2d(FAKE, FAKE, ipe.IPE_BF16, 256, 16, 72, 1152, 1152, g, n, 2, 0.0, None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp_rope2d(FAKE, 48, 1152, FAKE, FAKE, FAKE, 16, 72, 1152, 1152, 1e4, 5, g, n, 2, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_vis_interp_plan(g, n, 2, 300, FAKE, FAKE, FAKE, None), ipe.IPE_EINVAL)


def test_error_message_is_thread_local_and_cleared():
    out = (F * 4)()
    assert L.ipe_rope_inv_freq(7, 1e4, out) == ipe.IPE_EINVAL
    assert b"even" in L.ipe_last_error()
    assert L.ipe_rope_inv_freq(8, 1e4, out) == ipe.IPE_OK
    assert L.ipe_last_error() == b""
