"""Python binding of libipe.so, the B200 interpolated-position-encoding library.

Argument marshalling only: each function checks that its tensors are on the
GPU, passes ``data_ptr()``, sizes, strides and the current CUDA stream to the
C entry point of the same name (``include/ipe.h``) and raises
``IpeError`` with the library's message on a non-OK status.  Every step of
the computation runs in the library's CUDA kernels; there is no other path.
PyTorch is used for device memory and streams only.

Build the library first: ``python interpolated_position_encoding_b200/build.py``.
"""
import ctypes
import os

import torch

from . import build as _build

_LIB_PATH = _build.LIB

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python interpolated_position_encoding_b200/build.py` "
        "(nvcc for sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(_LIB_PATH)

_P, _I, _I64, _D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double

_SIGS = {
    "ipe_last_error": (ctypes.c_char_p, []),
    "ipe_version": (_I, []),
    "ipe_kernel_arch": (_I, [_P, _P]),
    "ipe_device_status": (_I, [_P]),
    "ipe_debug_inject": (_I, [_I64, _I64]),
    "ipe_rope_inv_freq": (_I, [_I, _D, _P]),
    "ipe_mrope_axis_map": (_I, [_I, _P, _I, _P, _P]),
    "ipe_mrope_cos_sin": (_I, [_P, _I64, _P, _I, _P, _I, _P, _P, _P]),
    "ipe_apply_rotary_partial": (_I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, _I, _P]),
    "ipe_mrope_apply": (_I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, _I, _P, _I, _P]),
    "ipe_qk_norm_mrope": (_I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, ctypes.c_float, _P, _P, _I, _P, _I,
                               _P]),
    "ipe_apply_rotary_partial_hf": (_I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, _I, _P]),
    "ipe_mrope_apply_hf": (_I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, _I, _P, _I, _P]),
    "ipe_vis_pos_interp_hf": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _P]),
    "ipe_host_join": (_I, [_P]),
    "ipe_mrope_apply_host": (_I, [_P, _P, _P, _P, _I, _I64, _I, _I, _I, _P, _P, _I, _P, _I, _P, _P, _P, _I64, _I, _P]),
    "ipe_vis_rope2d_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _D, _P, _P, _I64, _I, _P]),
    "ipe_vis_pos_interp_host": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _I64, _I, _P]),
    "ipe_mrope_decode": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _I64, _I64, _I64, _P, _P, _P, _P, ctypes.c_float, _P,
                              _I, _P, _P, _I64, _I64, _P, _P]),
    "ipe_mrope_rope_index": (_I, [_P, _P, _I, _I64, _I64, _P, _I, _P, _I, _I, _I, _P, _P, _P, ctypes.c_size_t, _P]),
    "ipe_mrope_rope_index_workspace": (ctypes.c_size_t, [_I64, _I64, _I, _I]),
    "ipe_mrope_rope_index_static": (_I, [_P, _P, _I, _I64, _I64, _P, _I, _P, _I, _I, _I, _P, _P, _P]),
    "ipe_vis_interp_plan": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "ipe_vis_pos_interp": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _P]),
    "ipe_vis_rope2d": (_I, [_P, _P, _I, _I64, _I, _I, _I64, _I64, _P, _I, _I, _D, _P]),
    "ipe_vis_pos_interp_rope2d": (_I, [_P, _I, _I, _P, _P, _P, _I, _I, _I64, _I64, _D, _I, _P, _I, _I, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTS = tuple(_SIGS)

IPE_F32, IPE_BF16 = 0, 1
IPE_OK, IPE_EINVAL, IPE_EALIGN, IPE_ELIMIT, IPE_ECUDA, IPE_EDEVICE = 0, 1, 2, 3, 4, 5
_STATUS = {1: "IPE_EINVAL", 2: "IPE_EALIGN", 3: "IPE_ELIMIT", 4: "IPE_ECUDA", 5: "IPE_EDEVICE"}


class IpeError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def _check(rc):
    if rc != IPE_OK:
        raise IpeError(rc, _lib.ipe_last_error().decode())


def lib():
    """The loaded ctypes library (raw C entry points)."""
    return _lib


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return IPE_BF16
    if t.dtype == torch.float32:
        return IPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32")


def _cuda(t, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    return t


def _cuda_device(device):
    if torch.device(device).type != "cuda":
        raise TypeError(f"device must be a CUDA device, not {device!r} (the library has no CPU path)")
    return device


try:
    _raw_stream = torch._C._cuda_getCurrentRawStream
except AttributeError:  # pragma: no cover - older torch
    _raw_stream = None


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


# Small caches of host arrays passed by value (keys are immutable tuples).
_HOST_CACHE = {}


def _cached(key, make):
    v = _HOST_CACHE.get(key)
    if v is None:
        if len(_HOST_CACHE) > 256:
            _HOST_CACHE.clear()
        v = _HOST_CACHE[key] = make()
    return v


def _i32_host(values, n=None):
    values = tuple(int(v) for v in values)
    if n is not None and len(values) != n:
        raise ValueError(f"expected {n} values, got {len(values)}")
    return _cached(("i32",) + values, lambda: (ctypes.c_int32 * len(values))(*values))


def _grid_host(grid_thw):
    if isinstance(grid_thw, torch.Tensor):
        flat = tuple(grid_thw.detach().cpu().reshape(-1).tolist())
    else:
        flat = tuple(int(v) for g in grid_thw for v in (g if hasattr(g, "__len__") else [g]))
    if len(flat) % 3:
        raise ValueError("grid_thw must hold (t, h, w) triples")
    return _i32_host(flat), len(flat) // 3


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _row_stride(t, heads, head_dim, name):
    """Token stride of a [rows, heads, head_dim] view with contiguous heads."""
    if t.dim() != 3 or t.shape[1] != heads or t.shape[2] != head_dim:
        raise ValueError(f"{name} must be [rows, {heads}, {head_dim}], got {tuple(t.shape)}")
    if t.stride(2) != 1 or (heads > 1 and t.stride(1) != head_dim):
        raise ValueError(f"{name}: heads must be contiguous (strides {t.stride()})")
    return t.stride(0)


def device_status(stream=None):
    """Synchronise the stream and raise IpeError(IPE_EDEVICE) if a kernel gave up a bounded wait."""
    _check(_lib.ipe_device_status(_stream(stream)))


def kernel_arch():
    """(binaryVersion, ptxVersion) of a library kernel as loaded on the current device (100 = sm_100a)."""
    b, p = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.ipe_kernel_arch(ctypes.byref(b), ctypes.byref(p)))
    return b.value, p.value


def debug_inject(skip_tile=-1, wait_cycles=0):
    """Test hook: TMA rotation producers skip tile `skip_tile`; waits give up after `wait_cycles`."""
    _check(_lib.ipe_debug_inject(int(skip_tile), int(wait_cycles)))


# --------------------------------------------------------------------- text


def rope_inv_freq(rot_dim, theta):
    """Default RoPE inverse frequencies (fp32, computed on the host by the library)."""
    out = (ctypes.c_float * (rot_dim // 2))()
    _check(_lib.ipe_rope_inv_freq(int(rot_dim), float(theta), out))
    return torch.tensor(list(out), dtype=torch.float32)


def mrope_axis_map(half, section, interleaved=True, device="cuda", stream=None):
    """int8 [half]: axis (0 = T, 1 = H, 2 = W) of each frequency."""
    out = torch.empty(half, dtype=torch.int8, device=_cuda_device(device))
    _check(_lib.ipe_mrope_axis_map(int(half), _i32_host(section, 3), int(bool(interleaved)), _ptr(out),
                                   _stream(stream)))
    return out


def _inv_host(inv_freq):
    if isinstance(inv_freq, torch.Tensor):
        if inv_freq.is_cuda:
            raise TypeError("inv_freq must be a host tensor or sequence (it travels as a kernel parameter)")
        vals = tuple(inv_freq.detach().float().reshape(-1).tolist())
    else:
        vals = tuple(float(v) for v in inv_freq)
    arr = _cached(("inv",) + vals, lambda: (ctypes.c_float * len(vals))(*vals))
    return arr, len(vals)


def mrope_cos_sin(positions, inv_freq, section, interleaved=True, cos=None, sin=None, stream=None):
    """cos, sin fp32 [T, 2*half] from int32 positions [3, T]."""
    _cuda(positions, "positions")
    if positions.dtype != torch.int32 or positions.dim() != 2 or positions.shape[0] != 3 or not positions.is_contiguous():
        raise ValueError("positions must be a contiguous int32 [3, T] tensor")
    T = positions.shape[1]
    inv, half = _inv_host(inv_freq)
    if cos is None:
        cos = torch.empty(T, 2 * half, dtype=torch.float32, device=positions.device)
    if sin is None:
        sin = torch.empty(T, 2 * half, dtype=torch.float32, device=positions.device)
    for t, n in ((cos, "cos"), (sin, "sin")):
        _cuda(t, n)
        if t.dtype != torch.float32 or tuple(t.shape) != (T, 2 * half) or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous float32 [{T}, {2 * half}] tensor")
    _check(_lib.ipe_mrope_cos_sin(_ptr(positions), T, inv, half, _i32_host(section, 3), int(bool(interleaved)),
                                  _ptr(cos), _ptr(sin), _stream(stream)))
    return cos, sin


def _qk_args(q, k):
    _cuda(q, "q")
    _cuda(k, "k")
    ref = q if q is not None else k
    if ref is None:
        raise ValueError("q and k are both None")
    if q is not None and k is not None and q.dtype != k.dtype:
        raise TypeError("q and k must share a dtype")
    T, head_dim = ref.shape[0], ref.shape[2]
    hq = q.shape[1] if q is not None else 0
    hk = k.shape[1] if k is not None else 0
    qs = _row_stride(q, hq, head_dim, "q") if q is not None else 0
    ks = _row_stride(k, hk, head_dim, "k") if k is not None else 0
    if k is not None and k.shape[0] != T:
        raise ValueError("q and k must have the same number of rows")
    return _dtype_code(ref), T, hq, hk, head_dim, qs, ks


def _rounding(rounding):
    if rounding not in ("fp32", "hf"):
        raise ValueError('rounding must be "fp32" (one rounding at the end) or "hf" (the reference listings\' '
                         'rounding points)')
    return rounding == "hf"


def apply_rotary_partial(q, k, cos, sin, stream=None, rounding="fp32"):
    """In place: rotate_half rotation of the first cos.shape[1] channels of q [T, hq, D], k [T, hk, D]."""
    dt, T, hq, hk, D, qs, ks = _qk_args(q, k)
    for t, n in ((cos, "cos"), (sin, "sin")):
        _cuda(t, n)
        if t.dtype != torch.float32 or t.dim() != 2 or t.shape[0] != T or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous float32 [T, rot_dim] tensor")
    fn = _lib.ipe_apply_rotary_partial_hf if _rounding(rounding) else _lib.ipe_apply_rotary_partial
    _check(fn(_ptr(q), _ptr(k), dt, T, hq, hk, D, qs, ks, _ptr(cos), _ptr(sin), cos.shape[1], _stream(stream)))
    return q, k


def mrope_apply(q, k, positions, inv_freq, section, interleaved=True, stream=None, rounding="fp32"):
    """In place: fused multimodal RoPE of q [T, hq, D] and k [T, hk, D] (cos / sin stay in registers)."""
    dt, T, hq, hk, D, qs, ks = _qk_args(q, k)
    _cuda(positions, "positions")
    if positions.dtype != torch.int32 or tuple(positions.shape) != (3, T) or not positions.is_contiguous():
        raise ValueError("positions must be a contiguous int32 [3, T] tensor")
    inv, half = _inv_host(inv_freq)
    fn = _lib.ipe_mrope_apply_hf if _rounding(rounding) else _lib.ipe_mrope_apply
    _check(fn(_ptr(q), _ptr(k), dt, T, hq, hk, D, qs, ks, _ptr(positions), inv, 2 * half, _i32_host(section, 3),
              int(bool(interleaved)), _stream(stream)))
    return q, k


def qk_norm_mrope(q, k, q_weight, k_weight, positions, inv_freq, section, interleaved=True, eps=1e-6, stream=None):
    """In place: RMSNorm of every head row (cast back, then the weight) and the
    fused multimodal rotation of its first 2 * len(inv_freq) channels."""
    dt, T, hq, hk, D, qs, ks = _qk_args(q, k)
    for w, nm in ((q_weight, "q_weight"), (k_weight, "k_weight")):
        _cuda(w, nm)
        ref = q if q is not None else k
        if w.dtype != ref.dtype or tuple(w.shape) != (D,) or not w.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous [{D}] tensor of the activation dtype")
    _cuda(positions, "positions")
    if positions.dtype != torch.int32 or tuple(positions.shape) != (3, T) or not positions.is_contiguous():
        raise ValueError("positions must be a contiguous int32 [3, T] tensor")
    inv, half = _inv_host(inv_freq)
    _check(_lib.ipe_qk_norm_mrope(_ptr(q), _ptr(k), dt, T, hq, hk, D, qs, ks, _ptr(q_weight), _ptr(k_weight),
                                  float(eps), _ptr(positions), inv, 2 * half, _i32_host(section, 3),
                                  int(bool(interleaved)), _stream(stream)))
    return q, k


def mrope_decode(q, k, seq_pos, inv_freq, rope_deltas=None, v=None, q_weight=None, k_weight=None, eps=1e-6,
                 k_cache=None, v_cache=None, slot_mapping=None, stream=None):
    """One generation step, in place: q [B, hq, D] and k [B, hk, D] (any
    token stride, contiguous heads) rotated at positions seq_pos + rope_deltas
    (int32 [B] each), after an optional QK-RMSNorm (q_weight, k_weight); with
    slot_mapping (int64 [B], < 0 = skip) the rotated k rows and the v rows are
    written to k_cache / v_cache ([num_slots, hk, D] views, any slot stride)."""
    dt, B, hq, hk, D, qs, ks = _qk_args(q, k)
    for t, nm in ((seq_pos, "seq_pos"), (rope_deltas, "rope_deltas")):
        if t is not None:
            _cuda(t, nm)
            if t.dtype != torch.int32 or tuple(t.shape) != (B,) or not t.is_contiguous():
                raise ValueError(f"{nm} must be a contiguous int32 [{B}] tensor")
    ref = q if q is not None else k
    for w, nm in ((q_weight, "q_weight"), (k_weight, "k_weight")):
        if w is not None:
            _cuda(w, nm)
            if w.dtype != ref.dtype or tuple(w.shape) != (D,) or not w.is_contiguous():
                raise ValueError(f"{nm} must be a contiguous [{D}] tensor of the activation dtype")
    vs = 0
    if v is not None:
        _cuda(v, "v")
        vs = _row_stride(v, hk, D, "v")
        if v.shape[0] != B or v.dtype != ref.dtype:
            raise ValueError("v must be [B, hk, D] of the activation dtype")
    cs, nslots = 0, 0
    if k_cache is not None:
        _cuda(k_cache, "k_cache")
        cs = _row_stride(k_cache, hk, D, "k_cache")
        nslots = k_cache.shape[0]
        if v_cache is not None:
            _cuda(v_cache, "v_cache")
            if _row_stride(v_cache, hk, D, "v_cache") != cs or v_cache.shape[0] != nslots:
                raise ValueError("v_cache must match k_cache in shape and slot stride")
    if slot_mapping is not None:
        _cuda(slot_mapping, "slot_mapping")
        if slot_mapping.dtype != torch.int64 or tuple(slot_mapping.shape) != (B,) or not slot_mapping.is_contiguous():
            raise ValueError(f"slot_mapping must be a contiguous int64 [{B}] tensor")
    inv, half = _inv_host(inv_freq)
    _check(_lib.ipe_mrope_decode(_ptr(q), _ptr(k), _ptr(v), dt, B, hq, hk, D, qs, ks, vs, _ptr(seq_pos),
                                 _ptr(rope_deltas), _ptr(q_weight), _ptr(k_weight), float(eps), inv, 2 * half,
                                 _ptr(k_cache), _ptr(v_cache), cs, nslots, _ptr(slot_mapping), _stream(stream)))
    return q, k


def rope_index_workspace_bytes(B, L, n_images=0, n_videos=0):
    """Device scratch bytes mrope_rope_index needs for these sizes."""
    n = _lib.ipe_mrope_rope_index_workspace(int(B), int(L), int(n_images), int(n_videos))
    if n == 0 and B > 0:
        raise ValueError(f"rope_index: sizes out of range (B={B}, L={L}, images={n_images}, videos={n_videos})")
    return n


def _int_tensor(t, name, shape=None):
    _cuda(t, name)
    if t.dtype not in (torch.int32, torch.int64) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 or int64 tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    return t


def mrope_rope_index(mm_token_type_ids, image_grid_thw=None, video_grid_thw=None, attention_mask=None,
                     spatial_merge_size=2, position_ids=None, rope_deltas=None, workspace=None, stream=None):
    """(position_ids int32 [3, B, L], rope_deltas int32 [B]) of a batch of
    mixed sequences, computed on the device.  Types and mask are [B, L] int32
    or int64 (the same dtype); grids [n, 3] int32 or int64 (the same dtype)."""
    ty = _int_tensor(mm_token_type_ids, "mm_token_type_ids")
    if ty.dim() != 2:
        raise ValueError("mm_token_type_ids must be [B, L]")
    B, L = ty.shape
    if attention_mask is not None:
        _int_tensor(attention_mask, "attention_mask", (B, L))
        if attention_mask.dtype != ty.dtype:
            raise ValueError("attention_mask must have the dtype of mm_token_type_ids")
    grids = [g for g in (image_grid_thw, video_grid_thw) if g is not None]
    for g, nm in zip(grids, ("grid",) * 2):
        _int_tensor(g, nm)
        if g.dim() != 2 or g.shape[1] != 3:
            raise ValueError("grids must be [n, 3]")
    if len(grids) == 2 and grids[0].dtype != grids[1].dtype:
        raise ValueError("image_grid_thw and video_grid_thw must share a dtype")
    gbytes = grids[0].element_size() if grids else 4
    n_img = 0 if image_grid_thw is None else image_grid_thw.shape[0]
    n_vid = 0 if video_grid_thw is None else video_grid_thw.shape[0]
    dev = ty.device
    if position_ids is None:
        position_ids = torch.empty(3, B, L, dtype=torch.int32, device=dev)
    if rope_deltas is None:
        rope_deltas = torch.empty(B, dtype=torch.int32, device=dev)
    for t, nm, shp in ((position_ids, "position_ids", (3, B, L)), (rope_deltas, "rope_deltas", (B,))):
        _cuda(t, nm)
        if t.dtype != torch.int32 or tuple(t.shape) != shp or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous int32 {shp} tensor")
    need = rope_index_workspace_bytes(B, L, n_img, n_vid) if B > 0 else 0
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _cuda(workspace, "workspace")
    _check(_lib.ipe_mrope_rope_index(_ptr(ty), _ptr(attention_mask), ty.element_size(), B, L, _ptr(image_grid_thw),
                                     n_img, _ptr(video_grid_thw), n_vid, gbytes, int(spatial_merge_size),
                                     _ptr(position_ids), _ptr(rope_deltas), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)))
    return position_ids, rope_deltas


# Bytes of the library-owned scratch behind mrope_rope_index_static (per device).
ROPE_INDEX_STATIC_BYTES = 4 << 20


def mrope_rope_index_static(mm_token_type_ids, image_grid_thw, video_grid_thw, attention_mask, spatial_merge_size,
                            position_ids, rope_deltas, stream=None):
    """mrope_rope_index for callers that cannot allocate device memory at call
    time: the outputs are the caller's, the scratch is a fixed buffer inside
    the library (ROPE_INDEX_STATIC_BYTES per device), and nothing is allocated
    here.  Calls on one device share that buffer, so calls that overlap in
    time race; the first call on a device does a one-time set-up and should
    come before any stream capture."""
    if not isinstance(mm_token_type_ids, torch.Tensor) or mm_token_type_ids.dim() != 2:
        raise ValueError("mm_token_type_ids must be a [B, L] tensor")
    B, L = mm_token_type_ids.shape
    n_img = 0 if image_grid_thw is None else image_grid_thw.shape[0]
    n_vid = 0 if video_grid_thw is None else video_grid_thw.shape[0]
    need = rope_index_workspace_bytes(B, L, n_img, n_vid)
    if need > ROPE_INDEX_STATIC_BYTES:
        raise IpeError(IPE_ELIMIT, f"these sizes need {need} bytes of scratch, above the {ROPE_INDEX_STATIC_BYTES} "
                                   "bytes of the library's fixed buffer")
    ty = _int_tensor(mm_token_type_ids, "mm_token_type_ids")
    if attention_mask is not None:
        _int_tensor(attention_mask, "attention_mask", (B, L))
    grids = [g for g in (image_grid_thw, video_grid_thw) if g is not None]
    for g in grids:
        _int_tensor(g, "grid")
    gbytes = grids[0].element_size() if grids else 4
    for t, nm, shp in ((position_ids, "position_ids", (3, B, L)), (rope_deltas, "rope_deltas", (B,))):
        _cuda(t, nm)
        if t.dtype != torch.int32 or tuple(t.shape) != shp or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous int32 {shp} tensor")
    _check(_lib.ipe_mrope_rope_index_static(_ptr(ty), _ptr(attention_mask), ty.element_size(), B, L,
                                            _ptr(image_grid_thw), n_img, _ptr(video_grid_thw), n_vid, gbytes,
                                            int(spatial_merge_size), _ptr(position_ids), _ptr(rope_deltas),
                                            _stream(stream)))
    return position_ids, rope_deltas


# ------------------------------------------------------ host buffers


def _host(t, name):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous host tensor (page-locked for overlap)")
    return t


def _dev_like(t, host, name):
    _cuda(t, name)
    if t.numel() * t.element_size() < host.numel() * host.element_size() or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous device tensor at least the size of its host buffer")
    return t


def host_join(stream=None):
    """The stream waits for every copy back to the host enqueued so far."""
    _check(_lib.ipe_host_join(_stream(stream)))


def mrope_apply_host(q, k, positions, inv_freq, section, interleaved, q_dev, k_dev, positions_dev, q_out=None,
                     k_out=None, chunk_tokens=8192, join=True, stream=None):
    """mrope_apply on host tensors q [T, hq, D], k [T, hk, D], positions [3, T]
    (int32), streamed through the device buffers in chunks; results land in
    q_out / k_out (default: in place)."""
    _host(q, "q"), _host(k, "k"), _host(positions, "positions")
    q_out = q if q_out is None else _host(q_out, "q_out")
    k_out = k if k_out is None else _host(k_out, "k_out")
    T, hq, D = q.shape
    hk = k.shape[1]
    _dev_like(q_dev, q, "q_dev"), _dev_like(k_dev, k, "k_dev"), _dev_like(positions_dev, positions, "positions_dev")
    inv, half = _inv_host(inv_freq)
    _check(_lib.ipe_mrope_apply_host(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _dtype_code(q), T, hq, hk, D,
                                     _ptr(positions), inv, 2 * half, _i32_host(section, 3), int(bool(interleaved)),
                                     _ptr(q_dev), _ptr(k_dev), _ptr(positions_dev), int(chunk_tokens), int(bool(join)),
                                     _stream(stream)))
    return q_out, k_out


def vis_rope2d_host(q, k, grid_thw, q_dev, k_dev, merge=2, theta=1e4, q_out=None, k_out=None, chunk_rows=16384,
                    join=True, stream=None):
    """vis_rope2d on host tensors q / k [N, heads, head_dim], streamed in chunks."""
    _host(q, "q")
    q_out = q if q_out is None else _host(q_out, "q_out")
    if k is not None:
        _host(k, "k")
        k_out = k if k_out is None else _host(k_out, "k_out")
    g, n = _grid_host(grid_thw)
    _, heads, hd = q.shape
    _dev_like(q_dev, q, "q_dev")
    if k is not None:
        _dev_like(k_dev, k, "k_dev")
    _check(_lib.ipe_vis_rope2d_host(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _dtype_code(q), heads, hd, g, n,
                                    int(merge), float(theta), _ptr(q_dev), _ptr(k_dev) if k is not None else None,
                                    int(chunk_rows), int(bool(join)), _stream(stream)))
    return q_out, k_out


def vis_pos_interp_host(table, grid_thw, out, table_dev, out_dev, merge=2, chunk_rows=16384, join=True,
                        stream=None):
    """vis_pos_interp from a host table to a host output, streamed in chunks."""
    _host(table, "table"), _host(out, "out")
    g, n = _grid_host(grid_thw)
    G = int(round(table.shape[0] ** 0.5))
    _dev_like(table_dev, table, "table_dev"), _dev_like(out_dev, out, "out_dev")
    _check(_lib.ipe_vis_pos_interp_host(_ptr(table), _dtype_code(table), G, table.shape[1], g, n, int(merge),
                                        _ptr(out), _ptr(table_dev), _ptr(out_dev), int(chunk_rows), int(bool(join)),
                                        _stream(stream)))
    return out


# ------------------------------------------------------------------- vision


def vis_interp_plan(grid_thw, merge=2, grid_side=48, device="cuda", stream=None):
    """(idx4 int32 [4, N], w4 float32 [4, N], rowcol int32 [2, N]) in output order."""
    g, n = _grid_host(grid_thw)
    N = sum(g[3 * i] * g[3 * i + 1] * g[3 * i + 2] for i in range(n))
    device = _cuda_device(device)
    idx4 = torch.empty(4, N, dtype=torch.int32, device=device)
    w4 = torch.empty(4, N, dtype=torch.float32, device=device)
    rowcol = torch.empty(2, N, dtype=torch.int32, device=device)
    _check(_lib.ipe_vis_interp_plan(g, n, int(merge), int(grid_side), _ptr(idx4), _ptr(w4), _ptr(rowcol),
                                    _stream(stream)))
    return idx4, w4, rowcol


def _table_args(table):
    _cuda(table, "table")
    if table.dim() != 2 or not table.is_contiguous():
        raise ValueError("table must be a contiguous [G*G, hidden] tensor")
    G = int(round(table.shape[0] ** 0.5))
    if G * G != table.shape[0]:
        raise ValueError("table rows must be a square grid G*G")
    return G, table.shape[1]


def vis_pos_interp(table, grid_thw, merge=2, out=None, stream=None, rounding="fp32"):
    """[N, hidden] interpolated position embeddings in merge order, dtype of the table."""
    G, C = _table_args(table)
    g, n = _grid_host(grid_thw)
    N = sum(g[3 * i] * g[3 * i + 1] * g[3 * i + 2] for i in range(n))
    if out is None:
        out = torch.empty(N, C, dtype=table.dtype, device=table.device)
    _cuda(out, "out")
    if out.dtype != table.dtype or tuple(out.shape) != (N, C) or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous [{N}, {C}] tensor of the table's dtype")
    fn = _lib.ipe_vis_pos_interp_hf if _rounding(rounding) else _lib.ipe_vis_pos_interp
    _check(fn(_ptr(table), _dtype_code(table), G, C, g, n, int(merge), _ptr(out), _stream(stream)))
    return out


def vis_rope2d(q, k, grid_thw, merge=2, theta=1e4, stream=None):
    """In place: vision 2-D rotary of q, k [N, heads, head_dim] (k may be None)."""
    _cuda(q, "q")
    _cuda(k, "k")
    heads, D = q.shape[1], q.shape[2]
    qs = _row_stride(q, heads, D, "q")
    ks = _row_stride(k, heads, D, "k") if k is not None else 0
    if k is not None and (k.dtype != q.dtype or k.shape[0] != q.shape[0]):
        raise ValueError("k must match q in dtype and rows")
    g, n = _grid_host(grid_thw)
    _check(_lib.ipe_vis_rope2d(_ptr(q), _ptr(k), _dtype_code(q), q.shape[0], heads, D, qs, ks, g, n, int(merge),
                               float(theta), _stream(stream)))
    return q, k


def vis_pos_interp_rope2d(table, grid_thw, q, k, merge=2, theta=1e4, out=None, stream=None):
    """Interpolated position embeddings (returned) and in-place 2-D rotary of q, k in one call, the two
    kernels running concurrently."""
    G, C = _table_args(table)
    g, n = _grid_host(grid_thw)
    N = sum(g[3 * i] * g[3 * i + 1] * g[3 * i + 2] for i in range(n))
    if out is None:
        out = torch.empty(N, C, dtype=table.dtype, device=table.device)
    _cuda(out, "out")
    _cuda(q, "q")
    _cuda(k, "k")
    if out.dtype != table.dtype or q.dtype != table.dtype or (k is not None and k.dtype != table.dtype):
        raise TypeError("table, out, q and k must share a dtype")
    if tuple(out.shape) != (N, C) or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous [{N}, {C}] tensor")
    heads, D = q.shape[1], q.shape[2]
    qs = _row_stride(q, heads, D, "q")
    ks = _row_stride(k, heads, D, "k") if k is not None else 0
    _check(_lib.ipe_vis_pos_interp_rope2d(_ptr(table), G, C, _ptr(out), _ptr(q), _ptr(k), heads, D, qs, ks,
                                          float(theta), _dtype_code(table), g, n, int(merge), _stream(stream)))
    return out, q, k


__all__ = ["IpeError", "lib", "EXPORTS", "device_status", "kernel_arch", "debug_inject", "rope_inv_freq", "mrope_axis_map", "mrope_cos_sin", "apply_rotary_partial",
           "mrope_apply", "qk_norm_mrope", "vis_interp_plan", "vis_pos_interp", "vis_rope2d", "vis_pos_interp_rope2d"]
