"""Transfers and the tolerance model of the GPU parity tests.

Tolerances (fixed for every test):
  fp32 outputs  |gpu - oracle| <= 2e-6 (absolute), the oracle in double;
  bf16 outputs  |gpu - oracle| <= ulp_bf16(oracle) + 2^-22 * mag, where mag is
                the sum of the magnitudes of the terms the output adds
                (|x_a cos| + |x_b sin| for a rotation, sum_c |w_c v_c| for the
                interpolation).  The second term covers fp32 evaluation near
                cancellation; away from it the bound is one bf16 ulp of the
                fp32-computed value cast once.
"""
import numpy as np
import torch

import workloads as wl

F32_ATOL = 2e-6
MAG_REL = 2.0 ** -22


def bf16_to_gpu(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def f32_to_gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def gpu_to_f64(t):
    if t.dtype == torch.bfloat16:
        bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        return wl.bf16_bits_to_f32(bits).astype(np.float64)
    return t.detach().float().cpu().numpy().astype(np.float64)


def host_f64(a, dtype):
    """Exact float64 of a workload tensor (fp32 array or bf16 bit patterns)."""
    return (wl.bf16_bits_to_f32(a) if dtype == "bf16" else np.asarray(a, np.float32)).astype(np.float64)


def to_gpu(a, dtype):
    return bf16_to_gpu(a) if dtype == "bf16" else f32_to_gpu(a)


def ulp_bf16(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def check(got, ref, mag, dtype, what):
    """Assert the tolerance; returns a small report dict."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        worst = float(err.max()) if err.size else 0.0
        assert worst <= F32_ATOL, f"{what}: max |err| {worst:.3e} > {F32_ATOL}"
        return {"max_abs": worst}
    ulp = ulp_bf16(ref)
    tol = ulp + MAG_REL * np.asarray(mag, np.float64)
    bad = err > tol
    if bad.any():
        i = int(np.argmax(err - tol))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst got "
                             f"{got.flat[i]!r} ref {ref.flat[i]!r} mag {np.asarray(mag).flat[i]!r}")
    return {"max_ulp": float((err / ulp).max()) if err.size else 0.0,
            "beyond_1ulp": int((err > ulp).sum())}
