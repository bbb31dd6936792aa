"""Shared helpers of the GPU parity tests: upload seeded inputs, compare with tolerances."""
from __future__ import annotations

import numpy as np
import torch

BF16_REL = 2.0 ** -8   # one bf16 ulp relative to the value (round-to-nearest is half of it)
F16_REL = 2.0 ** -10   # one fp16 ulp relative to the value


def torch_dtype(kind: str):
    return torch.bfloat16 if kind == "bf16" else torch.float32


def upload(inp, device="cuda"):
    """z, mask and weights of a TriMulInputs on the GPU in the storage dtype."""
    dt = torch_dtype(inp.dtype)
    z = torch.from_numpy(inp.z).to(device=device).to(dt)
    mask = torch.from_numpy(inp.mask).to(device=device).to(dt)
    w = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device=device).to(dt) for k, v in inp.weights.items()}
    return z, mask, w


def rms(x):
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def max_err_ratio(got, ref):
    """max |got - ref| / RMS(ref) over all entries."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    r = rms(ref)
    return float(np.max(np.abs(got - ref)) / r) if r > 0 else float(np.max(np.abs(got - ref)))


def assert_close_rms(got, ref, tol, what=""):
    ratio = max_err_ratio(got, ref)
    assert ratio <= tol, f"{what}: max|err| / RMS = {ratio:.3e} > {tol:.1e}"
    return ratio


def assert_close_ulp(got, ref, rms_tol, rel=BF16_REL, what=""):
    """Elementwise |got - ref| <= rel * |ref| + rms_tol * RMS(ref) (results stored in a 16-bit type;
    rel is one ulp of that type relative to the value)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    bound = rel * np.abs(ref) + rms_tol * rms(ref)
    bad = np.abs(got - ref) > bound
    if bad.any():
        i = np.unravel_index(np.argmax(np.abs(got - ref) - bound), ref.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} entries out of bound; worst at {i}: got {got[i]}, ref {ref[i]}")


def to_pair_major(t: torch.Tensor) -> np.ndarray:
    """[B, C, N, N] device tensor -> [B, N, N, C] float64 numpy."""
    return t.float().permute(0, 2, 3, 1).contiguous().cpu().numpy().astype(np.float64)


def assert_close_bf16(got, ref, rms_tol, what=""):
    assert_close_ulp(got, ref, rms_tol, BF16_REL, what)


def assert_close_f16(got, ref, rms_tol, what=""):
    assert_close_ulp(got, ref, rms_tol, F16_REL, what)
