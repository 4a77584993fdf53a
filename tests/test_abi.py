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


# ------------------------------------------------ entry points around the path
def test_rope_index_workspace_sizes():
    ws = L.ipe_mrope_rope_index_workspace
    assert ws(-1, 16, 0, 0) == 0 and ws(1, -1, 0, 0) == 0
    assert ws(1, (1 << 30) + 1, 0, 0) == 0                # L above 2^30
    assert ws(1 << 20, 1 << 12, 0, 0) == 0                # B * L above 2^31 - 1
    assert ws(1, 16, 16385, 0) == 0 and ws(1, 16, 0, -1) == 0
    small, large = ws(2, 4096, 3, 1), ws(2, 65536, 3, 1)
    assert 0 < small < large


def _ri(id_bytes=4, B=1, Lx=16, n_img=0, n_vid=0, grid_bytes=4, merge=2, types=FAKE, ws_bytes=1 << 20):
    return L.ipe_mrope_rope_index(types, None, id_bytes, B, Lx, FAKE if n_img else None, n_img,
                                  FAKE if n_vid else None, n_vid, grid_bytes, merge, FAKE, FAKE, FAKE, ws_bytes, None)


def test_rope_index_rejects():
    _err(_ri(id_bytes=2), ipe.IPE_EINVAL)
    _err(_ri(grid_bytes=3), ipe.IPE_EINVAL)
    _err(_ri(merge=0), ipe.IPE_EINVAL)
    _err(_ri(merge=65), ipe.IPE_EINVAL)
    _err(_ri(B=-1), ipe.IPE_EINVAL)
    _err(_ri(Lx=(1 << 30) + 1), ipe.IPE_ELIMIT)
    _err(_ri(n_img=16385), ipe.IPE_ELIMIT)
    need = L.ipe_mrope_rope_index_workspace(1, 16, 0, 0)
    _err(_ri(ws_bytes=need - 1), ipe.IPE_EINVAL)
    _err(_ri(types=ctypes.c_void_p(0x1002)), ipe.IPE_EALIGN)      # int32 ids on a 2-byte boundary
    assert _ri(B=0) == ipe.IPE_OK                                 # nothing to do, no device access


def _dec(head_dim=128, rot=64, invf=None, qw=FAKE, kw=FAKE, eps=1e-6, k_cache=FAKE, v_cache=FAKE, v=FAKE,
         cache_stride=256, num_slots=100, slots=FAKE, q=FAKE, B=4, hk=2):
    invf = inv(rot // 2) if invf is None else invf
    return L.ipe_mrope_decode(q, FAKE, v, ipe.IPE_BF16, B, 8, hk, head_dim, 8 * head_dim, hk * head_dim,
                              hk * head_dim, FAKE, None, qw, kw, eps, invf, rot, k_cache, v_cache, cache_stride,
                              num_slots, slots, None)


def test_decode_rejects():
    _err(_dec(head_dim=100), ipe.IPE_EINVAL)                      # not a multiple of 8 bf16
    _err(_dec(head_dim=8, rot=8), ipe.IPE_ELIMIT)                 # one chunk per row
    _err(_dec(rot=63), ipe.IPE_EINVAL)
    _err(_dec(rot=8), ipe.IPE_EINVAL)                             # rot / 2 not a multiple of 8
    bad = inv(32)
    bad[5] = float("inf")
    _err(_dec(invf=bad), ipe.IPE_EINVAL)
    _err(_dec(kw=None), ipe.IPE_EINVAL)                           # one norm weight only
    _err(_dec(eps=-1.0), ipe.IPE_EINVAL)
    _err(_dec(slots=None), ipe.IPE_EINVAL)                        # caches without slot_mapping
    _err(_dec(k_cache=None), ipe.IPE_EINVAL)                      # slot_mapping without k_cache
    _err(_dec(v=None), ipe.IPE_EINVAL)                            # v_cache without v
    _err(_dec(cache_stride=255), ipe.IPE_EINVAL)
    _err(_dec(num_slots=-1), ipe.IPE_EINVAL)
    _err(_dec(B=0, q=ctypes.c_void_p(0x1008)), ipe.IPE_EALIGN)    # q not 16-byte aligned
    assert _dec(B=0) == ipe.IPE_OK
    # no norm and no cache: weights, caches and slot_mapping all NULL
    assert _dec(B=0, qw=None, kw=None, k_cache=None, v_cache=None, slots=None) == ipe.IPE_OK


def _qkn(head_dim=128, rot=64, eps=1e-6, s=(11, 11, 10), qw=FAKE, T=16, q=FAKE):
    return L.ipe_qk_norm_mrope(q, FAKE, ipe.IPE_BF16, T, 8, 2, head_dim, 8 * head_dim, 2 * head_dim, qw, FAKE,
                               eps, FAKE, inv(rot // 2), rot, sec(*s), 1, None)


def test_qk_norm_rejects():
    _err(_qkn(head_dim=100), ipe.IPE_EINVAL)
    _err(_qkn(head_dim=8, rot=8, s=(4, 0, 0)), ipe.IPE_ELIMIT)    # one chunk per row
    _err(_qkn(head_dim=512, rot=64), ipe.IPE_ELIMIT)              # 64 chunks per row
    _err(_qkn(rot=63, s=(11, 11, 9)), ipe.IPE_EINVAL)
    _err(_qkn(rot=8, s=(2, 1, 1)), ipe.IPE_EINVAL)                # rot / 2 not a multiple of 8
    _err(_qkn(eps=float("nan")), ipe.IPE_EINVAL)
    _err(_qkn(eps=-1e-6), ipe.IPE_EINVAL)
    _err(_qkn(s=(11, 11, 9)), ipe.IPE_EINVAL)                     # section does not sum to rot / 2
    _err(_qkn(T=0, qw=ctypes.c_void_p(0x1004)), ipe.IPE_EALIGN)
    _err(_qkn(T=0, q=ctypes.c_void_p(0x1008)), ipe.IPE_EALIGN)
    assert _qkn(T=0) == ipe.IPE_OK


def test_hf_entry_points_reject():
    g, n = grid((1, 16, 16))
    _err(L.ipe_vis_pos_interp_hf(FAKE, ipe.IPE_BF16, 48, 1148, g, n, 2, FAKE, None), ipe.IPE_EINVAL)  # hidden % 8
    _err(L.ipe_vis_pos_interp_hf(ctypes.c_void_p(0x1008), ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, None),
         ipe.IPE_EALIGN)
    _err(L.ipe_vis_pos_interp_hf(FAKE, 9, 48, 1152, g, n, 2, FAKE, None), ipe.IPE_EINVAL)
    g0, n0 = grid((1, 15, 16))
    _err(L.ipe_vis_pos_interp_hf(FAKE, ipe.IPE_BF16, 48, 1152, g0, n0, 2, FAKE, None), ipe.IPE_EINVAL)
    _err(L.ipe_mrope_apply_hf(FAKE, FAKE, ipe.IPE_BF16, 16, 24, 4, 256, 6144, 1024, FAKE, inv(32), 64,
                              sec(11, 10, 10), 1, None), ipe.IPE_EINVAL)
    _err(L.ipe_apply_rotary_partial_hf(FAKE, FAKE, ipe.IPE_BF16, 8, 2, 2, 16, 32, 32, FAKE, FAKE, 5, None),
         ipe.IPE_EINVAL)


def test_host_entry_points_reject():
    # ipe_mrope_apply_host: chunk size, sizes, missing buffers
    def mah(chunk=4096, T=16, qh=FAKE, pos=FAKE):
        return L.ipe_mrope_apply_host(qh, FAKE, qh, FAKE, ipe.IPE_BF16, T, 24, 4, 256, pos, inv(32), 64,
                                      sec(11, 11, 10), 1, FAKE, FAKE, FAKE, chunk, 1, None)
    _err(mah(chunk=0), ipe.IPE_EINVAL)
    _err(mah(T=-1), ipe.IPE_EINVAL)
    _err(mah(qh=None), ipe.IPE_EINVAL)
    _err(mah(pos=None), ipe.IPE_EINVAL)
    g, n = grid((1, 16, 16))
    gz, nz = grid((1, 0, 16))
    _err(L.ipe_vis_rope2d_host(FAKE, FAKE, FAKE, FAKE, ipe.IPE_BF16, 16, 72, g, n, 2, 1e4, FAKE, FAKE, 0, 1, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_vis_rope2d_host(FAKE, FAKE, FAKE, FAKE, ipe.IPE_BF16, 16, 72, gz, nz, 2, 1e4, FAKE, FAKE, 64, 1,
                               None), ipe.IPE_EINVAL)
    _err(L.ipe_vis_rope2d_host(None, FAKE, FAKE, FAKE, ipe.IPE_BF16, 16, 72, g, n, 2, 1e4, FAKE, FAKE, 64, 1, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp_host(FAKE, ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, FAKE, FAKE, 0, 1, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp_host(FAKE, ipe.IPE_BF16, 48, 1152, gz, nz, 2, FAKE, FAKE, FAKE, 64, 1, None),
         ipe.IPE_EINVAL)
    _err(L.ipe_vis_pos_interp_host(FAKE, ipe.IPE_BF16, 48, 1152, g, n, 2, FAKE, None, FAKE, 64, 1, None),
         ipe.IPE_EINVAL)
