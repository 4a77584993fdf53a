"""Double-precision CPU oracle for the positional-encoding path (numpy front end).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package; the CUDA library and its binding
never do.  The arithmetic lives in ``oracle.c`` (see its header for the pages
and sections each function follows); this module only marshals numpy arrays.

All floating-point results are float64.  Inputs that the method defines in
fp32 (inverse frequencies) are float32; integer inputs are int32/int64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Bindings to one build of ``oracle.c`` (the default build, or a test variant)."""

    def __init__(self, lib_path=None):
        if lib_path is None:
            lib_path = _build.build()
        self.lib_path = lib_path
        lib = ctypes.CDLL(lib_path)
        sig = {
            "orc_rope_inv_freq": (_I, [_I, _D, _P]),
            "orc_mrope_axis_labels": (_I, [_I, _P, _I, _P]),
            "orc_mrope_cos_sin": (_I, [_P, _I64, _P, _I, _P, _I, _P, _P]),
            "orc_rotate_half": (None, [_P, _I, _P]),
            "orc_apply_rotary": (_I, [_P, _I64, _I, _I, _P, _P, _I, _P, _P]),
            "orc_grid_patches": (_I64, [_P, _I, _I]),
            "orc_vis_pos_embed_interpolate": (_I, [_P, _I, _I, _P, _I, _I, _P, _P]),
            "orc_vis_interp_plan": (_I, [_P, _I, _I, _I, _P, _P]),
            "orc_vis_rot_pos_ids": (_I, [_P, _I, _I, _P]),
            "orc_vis_rotary_cos_sin": (_I, [_P, _I64, _I, _D, _P, _P]),
            "orc_rms_norm": (_I, [_P, _I64, _I, _P, _D, _I, _P]),
            "orc_rope_index": (_I, [_P, _P, _I, _I64, _P, _I, _P, _I, _I, _P, _P]),
            "orc_decode_positions": (_I, [_P, _I, _I64, _P, _I64, _P, _P]),
            "orc_vis_pos_interp_hf": (_I, [_P, _I, _I, _P, _I, _I, _P, _P, _I, _P]),
            "orc_apply_rotary_hf": (_I, [_P, _I64, _I, _I, _P, _P, _I, _I, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        self._lib = lib

    # ---------------------------------------------------------------- text
    def rope_inv_freq(self, dim, base):
        out = np.zeros((dim + 1) // 2, np.float32)
        n = self._lib.orc_rope_inv_freq(int(dim), float(base), _ptr(out))
        if n < 0:
            raise ValueError("rope_inv_freq: bad arguments")
        return out

    def mrope_axis_labels(self, half, section, interleaved):
        sec = np.ascontiguousarray(section, np.int32)
        out = np.zeros(half, np.int32)
        if self._lib.orc_mrope_axis_labels(int(half), _ptr(sec), int(bool(interleaved)), _ptr(out)):
            raise ValueError("mrope_axis_labels: section must be 3 non-negative counts summing to half")
        return out

    def mrope_cos_sin(self, positions, inv_freq, section, interleaved):
        pos = np.ascontiguousarray(positions, np.int64)
        assert pos.ndim == 2 and pos.shape[0] == 3
        T = pos.shape[1]
        inv = np.ascontiguousarray(inv_freq, np.float32)
        half = inv.shape[0]
        sec = np.ascontiguousarray(section, np.int32)
        cos = np.zeros((T, 2 * half), np.float64)
        sin = np.zeros((T, 2 * half), np.float64)
        rc = self._lib.orc_mrope_cos_sin(_ptr(pos), T, _ptr(inv), half, _ptr(sec),
                                         int(bool(interleaved)), _ptr(cos), _ptr(sin))
        if rc:
            raise ValueError("mrope_cos_sin: bad arguments")
        return cos, sin

    def rotate_half(self, x):
        x = np.ascontiguousarray(x, np.float64)
        out = np.zeros_like(x)
        self._lib.orc_rotate_half(_ptr(x), x.shape[-1], _ptr(out))
        return out

    def apply_rotary(self, x, cos, sin, with_mag=False):
        """x: [T, H, D]; cos, sin: [T, rot] -> out [T, H, D] (and mag [T, H, rot])."""
        x = np.ascontiguousarray(x, np.float64)
        cos = np.ascontiguousarray(cos, np.float64)
        sin = np.ascontiguousarray(sin, np.float64)
        T, H, D = x.shape
        rot = cos.shape[1]
        assert cos.shape == (T, rot) and sin.shape == (T, rot)
        out = np.zeros_like(x)
        mag = np.zeros((T, H, rot), np.float64) if with_mag else None
        rc = self._lib.orc_apply_rotary(_ptr(x), T, H, D, _ptr(cos), _ptr(sin), rot, _ptr(out),
                                        _ptr(mag) if with_mag else None)
        if rc:
            raise ValueError("apply_rotary: bad arguments")
        return (out, mag) if with_mag else out

    def mrope_apply(self, x, positions, inv_freq, section, interleaved, with_mag=False):
        cos, sin = self.mrope_cos_sin(positions, inv_freq, section, interleaved)
        return self.apply_rotary(x, cos, sin, with_mag)

    def rms_norm(self, x, weight, eps, dtype):
        """RMSNorm over the last axis: x [..., D] -> rounded to `dtype` ("f32" | "bf16")."""
        x = np.ascontiguousarray(x, np.float64)
        w = np.ascontiguousarray(weight, np.float64)
        D = x.shape[-1]
        assert w.shape == (D,)
        out = np.zeros_like(x)
        R = x.size // D
        if self._lib.orc_rms_norm(_ptr(x), R, D, _ptr(w), float(eps), {"f32": 0, "bf16": 1}[dtype], _ptr(out)):
            raise ValueError("rms_norm: bad arguments")
        return out

    def qk_norm_mrope(self, x, weight, eps, dtype, positions, inv_freq, section, interleaved, with_mag=False):
        """RMSNorm of every head row, then the multimodal rotation of its first
        2 * len(inv_freq) channels (x: [T, H, D])."""
        y = self.rms_norm(x, weight, eps, dtype)
        out = self.mrope_apply(y, positions, inv_freq, section, interleaved, with_mag)
        return (out[0], out[1], y) if with_mag else (out, y)

    def rope_index(self, types, mask, image_grid_thw, video_grid_thw, merge):
        """(position_ids [3, B, L], rope_deltas [B]) of a batch of mixed
        sequences (types [B, L]; mask [B, L] or None; grids [n, 3] or None)."""
        ty = np.ascontiguousarray(types, np.int64)
        assert ty.ndim == 2
        B, L = ty.shape
        mk = None if mask is None else np.ascontiguousarray(mask, np.int64)
        assert mk is None or mk.shape == ty.shape
        ig = np.ascontiguousarray(np.zeros((0, 3)) if image_grid_thw is None else image_grid_thw, np.int64).reshape(-1, 3)
        vg = np.ascontiguousarray(np.zeros((0, 3)) if video_grid_thw is None else video_grid_thw, np.int64).reshape(-1, 3)
        pos = np.zeros((3, B, L), np.int64)
        deltas = np.zeros(B, np.int64)
        rc = self._lib.orc_rope_index(_ptr(ty), None if mk is None else _ptr(mk), B, L, _ptr(ig), ig.shape[0],
                                      _ptr(vg), vg.shape[0], int(merge), _ptr(pos), _ptr(deltas))
        if rc == -2:
            raise ValueError("rope_index: a vision run found its grid iterator exhausted")
        if rc == -3:
            raise ValueError("rope_index: the joined table does not have one column per kept slot")
        if rc:
            raise ValueError("rope_index: bad arguments")
        return pos, deltas

    def decode_positions(self, n_new, mask=None, cache_len=None, deltas=None):
        """Positions [3, B, n_new] of the newest n_new tokens of each sample,
        from the padding mask [B, S] (or the cache lengths [B]) and the rope
        deltas [B]."""
        mk = None if mask is None else np.ascontiguousarray(mask, np.int64)
        cl = None if cache_len is None else np.ascontiguousarray(cache_len, np.int64)
        B = mk.shape[0] if mk is not None else cl.shape[0]
        S = mk.shape[1] if mk is not None else 0
        dl = None if deltas is None else np.ascontiguousarray(deltas, np.int64)
        pos = np.zeros((3, B, n_new), np.int64)
        if self._lib.orc_decode_positions(None if mk is None else _ptr(mk), B, S, None if cl is None else _ptr(cl),
                                          int(n_new), None if dl is None else _ptr(dl), _ptr(pos)):
            raise ValueError("decode_positions: bad arguments")
        return pos

    # ------------------------------------------------------ HF rounding
    def apply_rotary_hf(self, x, cos32, sin32, dtype):
        """x [T, H, D] (values of `dtype`), cos / sin fp32 [T, rot]: the
        rotation with every product and sum rounded to `dtype`."""
        x = np.ascontiguousarray(x, np.float64)
        c = np.ascontiguousarray(cos32, np.float32)
        s_ = np.ascontiguousarray(sin32, np.float32)
        T, H, D = x.shape
        out = np.zeros_like(x)
        if self._lib.orc_apply_rotary_hf(_ptr(x), T, H, D, _ptr(c), _ptr(s_), c.shape[1], {"f32": 0, "bf16": 1}[dtype],
                                         _ptr(out)):
            raise ValueError("apply_rotary_hf: bad arguments")
        return out

    def mrope_cos_sin_f32(self, positions, inv_freq, section, interleaved):
        """The fp32 cos / sin tables: the double results rounded once."""
        cos, sin = self.mrope_cos_sin(positions, inv_freq, section, interleaved)
        return cos.astype(np.float32), sin.astype(np.float32)

    def mrope_apply_hf(self, x, positions, inv_freq, section, interleaved, dtype):
        cos, sin = self.mrope_cos_sin_f32(positions, inv_freq, section, interleaved)
        return self.apply_rotary_hf(x, cos, sin, dtype)

    @staticmethod
    def linspace_f32(G, n):
        """torch.linspace(0, G - 1, n) in fp32 (CPU), the listing's sample points."""
        import torch
        return torch.linspace(0, G - 1, n).numpy().astype(np.float32)

    def vis_pos_interp_hf(self, table, grid_thw, merge, dtype):
        """table [G*G, C] (values of `dtype`) -> [N, C] with the listing's
        rounding points (fp32 linspace, weights and products in the dtype,
        left-to-right sums)."""
        tab = np.ascontiguousarray(table, np.float64)
        GG, C = tab.shape
        G = int(round(GG ** 0.5))
        g = np.ascontiguousarray(grid_thw, np.int32).reshape(-1, 3)
        N = self.grid_patches(g, merge)
        ys = np.ascontiguousarray(np.concatenate([self.linspace_f32(G, int(h)) for _, h, _ in g] or [np.zeros(0)]),
                                  np.float32)
        xs = np.ascontiguousarray(np.concatenate([self.linspace_f32(G, int(w)) for _, _, w in g] or [np.zeros(0)]),
                                  np.float32)
        out = np.zeros((N, C), np.float64)
        if self._lib.orc_vis_pos_interp_hf(_ptr(tab), G, C, _ptr(g), g.shape[0], int(merge), _ptr(ys), _ptr(xs),
                                           {"f32": 0, "bf16": 1}[dtype], _ptr(out)):
            raise ValueError("vis_pos_interp_hf: bad arguments")
        return out

    # -------------------------------------------------------------- vision
    def grid_patches(self, grid_thw, merge):
        g = np.ascontiguousarray(grid_thw, np.int32).reshape(-1, 3)
        n = self._lib.orc_grid_patches(_ptr(g), g.shape[0], int(merge))
        if n < 0:
            raise ValueError("bad grid_thw / merge")
        return int(n)

    def vis_pos_embed_interpolate(self, table, grid_thw, merge, with_mag=False):
        """table: [G*G, C] -> [N, C] in merge order (and the |term| sums)."""
        tab = np.ascontiguousarray(table, np.float64)
        GG, C = tab.shape
        G = int(round(GG ** 0.5))
        assert G * G == GG
        g = np.ascontiguousarray(grid_thw, np.int32).reshape(-1, 3)
        N = self.grid_patches(g, merge)
        out = np.zeros((N, C), np.float64)
        mag = np.zeros((N, C), np.float64) if with_mag else None
        rc = self._lib.orc_vis_pos_embed_interpolate(_ptr(tab), G, C, _ptr(g), g.shape[0], int(merge),
                                                     _ptr(out), _ptr(mag) if with_mag else None)
        if rc:
            raise ValueError("vis_pos_embed_interpolate: bad arguments")
        return (out, mag) if with_mag else out

    def vis_interp_plan(self, grid_thw, merge, grid_side):
        g = np.ascontiguousarray(grid_thw, np.int32).reshape(-1, 3)
        N = self.grid_patches(g, merge)
        idx = np.zeros((4, N), np.int64)
        w = np.zeros((4, N), np.float64)
        if self._lib.orc_vis_interp_plan(_ptr(g), g.shape[0], int(merge), int(grid_side), _ptr(idx), _ptr(w)):
            raise ValueError("vis_interp_plan: bad arguments")
        return idx, w

    def vis_rot_pos_ids(self, grid_thw, merge):
        g = np.ascontiguousarray(grid_thw, np.int32).reshape(-1, 3)
        N = self.grid_patches(g, merge)
        out = np.zeros((N, 2), np.int64)
        if self._lib.orc_vis_rot_pos_ids(_ptr(g), g.shape[0], int(merge), _ptr(out)):
            raise ValueError("vis_rot_pos_ids: bad arguments")
        return out

    def vis_rotary_cos_sin(self, pos_ids, head_dim, theta):
        p = np.ascontiguousarray(pos_ids, np.int64)
        N = p.shape[0]
        cos = np.zeros((N, head_dim), np.float64)
        sin = np.zeros((N, head_dim), np.float64)
        if self._lib.orc_vis_rotary_cos_sin(_ptr(p), N, int(head_dim), float(theta), _ptr(cos), _ptr(sin)):
            raise ValueError("vis_rotary_cos_sin: bad arguments")
        return cos, sin

    def vis_apply_rotary(self, x, grid_thw, merge, theta, with_mag=False):
        """x: [N, heads, head_dim] -> 2-D rotary over the whole head."""
        x = np.ascontiguousarray(x, np.float64)
        pos_ids = self.vis_rot_pos_ids(grid_thw, merge)
        cos, sin = self.vis_rotary_cos_sin(pos_ids, x.shape[2], theta)
        return self.apply_rotary(x, cos, sin, with_mag)


_default = None


def get():
    """The oracle built from ``oracle.c`` as committed."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
