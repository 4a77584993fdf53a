"""Seeded synthetic inputs for the five positional-encoding workloads.

Shared by the tests, the benchmark and the smoke check; it holds none of the
method's arithmetic (no interpolation, frequencies, angles or rotation): only
random tensors, the fp32 -> bf16 round-to-nearest-even cast, image grids and
the position layout of a mixed text / image / video / audio sequence.

Position layout ("Interleaved Rotary Position Embedding", taking-lying-flat.github.io,
get_rope_index): a text run of n tokens takes cur .. cur + n - 1 on all three
rows and advances cur by n; a vision block of grid (t, h, w) patches (before
the m x m merge) places its merged tokens width-fastest at
(T, H, W) = (cur + frame, cur + row, cur + col) and advances cur by
max(h, w) / m.  Audio is linear in time, which for positions is a text run
("M01 RMSNorm and multimodal RoPE", problem summary).

bf16 tensors are numpy uint16 arrays of bf16 bit patterns.
"""
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------
# bf16 bit patterns
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x):
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32).copy()
    nan = np.isnan(x)
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    out = (u >> np.uint32(16)).astype(np.uint16)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(b):
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def rng_for(config_index, stream):
    """Generator of one (workload, tensor) pair: seed = 1000 + workload index."""
    return np.random.default_rng([1000 + int(config_index), int(stream)])


_CHUNK = 1 << 22


def _fill_normal(key, n, std, to_bf16):
    """N(0, std^2) samples, chunk c drawn from default_rng(key + (c,)), so the
    values do not depend on how many threads fill them."""
    out = np.empty(n, np.uint16 if to_bf16 else np.float32)

    def work(c):
        s, e = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        v = np.random.default_rng(list(key) + [c]).standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[s:e] = f32_to_bf16_bits(v) if to_bf16 else v

    nchunks = (n + _CHUNK - 1) // _CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def normal_f32(rng, shape, std=1.0):
    """N(0, std^2) in fp32.  rng: a numpy Generator, or a seed key (tuple of ints)."""
    n = int(np.prod(shape))
    if isinstance(rng, tuple):
        return _fill_normal(rng, n, std, False).reshape(shape)
    out = rng.standard_normal(n, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def normal_bf16(rng, shape, std=1.0):
    """N(0, std^2) drawn in fp32 and cast once (RNE) to bf16 bit patterns.
    rng: a numpy Generator, or a seed key (tuple of ints)."""
    n = int(np.prod(shape))
    if isinstance(rng, tuple):
        return _fill_normal(rng, n, std, True).reshape(shape)
    return f32_to_bf16_bits(normal_f32(rng, (n,), std)).reshape(shape)


# --------------------------------------------------------------------------
# Position layout of a mixed sequence
# --------------------------------------------------------------------------


def build_positions(segments, merge=2):
    """positions[3, T] (int32) for a list of segments.

    segments: ("text", n) | ("audio", n) | ("vision", (t, h, w)).
    Returns (positions, next_position) where next_position is the first
    position after the sequence.
    """
    rows = []
    cur = 0
    for kind, arg in segments:
        if kind in ("text", "audio"):
            n = int(arg)
            p = np.arange(cur, cur + n, dtype=np.int64)
            rows.append(np.stack([p, p, p]))
            cur += n
        elif kind == "vision":
            t, h, w = (int(v) for v in arg)
            if h % merge or w % merge:
                raise ValueError("grid not divisible by merge")
            gh, gw = h // merge, w // merge
            tt, hh, ww = np.meshgrid(np.arange(t), np.arange(gh), np.arange(gw), indexing="ij")
            rows.append(np.stack([tt.reshape(-1) + cur, hh.reshape(-1) + cur, ww.reshape(-1) + cur]))
            cur += max(h, w) // merge
        else:
            raise ValueError(f"unknown segment kind {kind!r}")
    if not rows:
        return np.zeros((3, 0), np.int32), 0
    pos = np.concatenate(rows, axis=1)
    return pos.astype(np.int32), cur


def segments_length(segments, merge=2):
    n = 0
    for kind, arg in segments:
        if kind in ("text", "audio"):
            n += int(arg)
        else:
            t, h, w = arg
            n += t * (h // merge) * (w // merge)
    return n


# --------------------------------------------------------------------------
# The five workloads
# --------------------------------------------------------------------------

VISION_GRID_CHOICES = [(1, 48, 64), (1, 32, 32), (1, 64, 96), (2, 28, 28), (1, 80, 56)]


@dataclass
class VisionSpec:
    grid_thw: list            # [(t, h, w), ...] before the merge
    dtype: str                # "f32" | "bf16" (table, q, k and output)
    merge: int = 2
    grid_side: int = 48
    hidden: int = 1152
    heads: int = 16
    head_dim: int = 72
    theta: float = 1e4
    table_std: float = 0.02
    fused: bool = False       # interpolation and 2-D rotary in one launch


@dataclass
class TextSpec:
    T: int
    hq: int
    hk: int
    head_dim: int
    rot_dim: int
    theta: float
    section: tuple
    layouts: tuple            # subset of ("interleaved", "chunked")
    segments: list = field(default_factory=list)
    merge: int = 2


@dataclass
class Workload:
    index: int                # 1-based; seeds are 1000 + index
    name: str
    vision: VisionSpec = None
    text: TextSpec = None


def _cfg3_segments():
    img = ("vision", (1, 32, 48))
    return [("text", 2048), img, ("text", 1024), img, ("text", 4096), ("audio", 8192),
            img, ("text", 2048), img, ("text", 13824)]


def _cfg5_segments(T=131072):
    segs = [("text", 8192)]
    for _ in range(16):
        segs += [("text", 6), ("vision", (1, 64, 64))]
    used = segments_length(segs)
    segs.append(("text", T - used))
    return segs


def key_for(config_index, stream):
    """Seed key of one (workload, tensor) pair: (1000 + workload index, stream)."""
    return (1000 + int(config_index), int(stream))


def _vision_batch8_grids():
    rng = rng_for(4, 5)
    pick = rng.integers(0, len(VISION_GRID_CHOICES), size=8)
    return [VISION_GRID_CHOICES[i] for i in pick]


WORKLOADS = {
    "vision_16x16_f32": Workload(
        1, "vision_16x16_f32",
        vision=VisionSpec(grid_thw=[(1, 16, 16)], dtype="f32")),
    "text_t4096_qwen35": Workload(
        2, "text_t4096_qwen35",
        text=TextSpec(T=4096, hq=24, hk=4, head_dim=256, rot_dim=64, theta=1e7,
                      section=(11, 11, 10), layouts=("interleaved",),
                      segments=[("text", 1024), ("vision", (1, 48, 64)), ("text", 2304)])),
    "text_t32768_omni": Workload(
        3, "text_t32768_omni",
        text=TextSpec(T=32768, hq=32, hk=4, head_dim=128, rot_dim=128, theta=1e6,
                      section=(24, 20, 20), layouts=("interleaved", "chunked"),
                      segments=_cfg3_segments())),
    "vision_batch8_bf16": Workload(
        4, "vision_batch8_bf16",
        vision=VisionSpec(grid_thw=_vision_batch8_grids(), dtype="bf16", fused=True)),
    "prefill_t131072_video": Workload(
        5, "prefill_t131072_video",
        vision=VisionSpec(grid_thw=[(16, 64, 64)], dtype="bf16"),
        text=TextSpec(T=131072, hq=24, hk=4, head_dim=256, rot_dim=64, theta=1e7,
                      section=(11, 11, 10), layouts=("interleaved",),
                      segments=_cfg5_segments())),
}

# Streams of key_for(index, stream)
S_TABLE, S_QV, S_KV, S_Q, S_K, S_GRID = 0, 1, 2, 3, 4, 5


def n_patches(vspec):
    return sum(t * h * w for t, h, w in vspec.grid_thw)


def vision_inputs(w):
    """dict(table [G*G, C], q [N, heads, head_dim], k, grid_thw int32 [n, 3]).

    f32 workloads give float32 arrays; bf16 workloads give uint16 bit patterns.
    """
    v = w.vision
    N = n_patches(v)
    gen = normal_f32 if v.dtype == "f32" else normal_bf16
    return {
        "table": gen(key_for(w.index, S_TABLE), (v.grid_side * v.grid_side, v.hidden), v.table_std),
        "q": gen(key_for(w.index, S_QV), (N, v.heads, v.head_dim)),
        "k": gen(key_for(w.index, S_KV), (N, v.heads, v.head_dim)),
        "grid_thw": np.asarray(v.grid_thw, np.int32).reshape(-1, 3),
    }


def text_inputs(w, with_qk=True):
    """dict(positions int32 [3, T], q bf16 [T, hq, D], k bf16 [T, hk, D])."""
    t = w.text
    pos, _ = build_positions(t.segments, t.merge)
    assert pos.shape[1] == t.T, (pos.shape, t.T)
    out = {"positions": pos}
    if with_qk:
        out["q"] = normal_bf16(key_for(w.index, S_Q), (t.T, t.hq, t.head_dim))
        out["k"] = normal_bf16(key_for(w.index, S_K), (t.T, t.hk, t.head_dim))
    return out
