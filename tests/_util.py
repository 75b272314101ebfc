"""Shared helpers of the test suite: device transfer and error metrics."""

from __future__ import annotations

import numpy as np
import torch

import synth


def rel_err(x, ref):
    """max |x - ref| / max |ref| over the whole tensor (normwise relative)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = max(float(np.max(np.abs(ref))), 1e-30)
    return float(np.max(np.abs(x - ref))) / den


def assert_close_elementwise(x, ref, rtol, atol, what=""):
    """Every element within |x - ref| <= rtol * |ref| + atol.

    This is the per-element form of a relative tolerance: a small element is
    held to its own magnitude, not to the largest element of the tensor
    (atol only covers reference values at or near zero)."""
    x = np.asarray(x, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert x.shape == ref.shape, (what, x.shape, ref.shape)
    if ref.size == 0:
        return
    assert np.all(np.isfinite(x) == np.isfinite(ref)), f"{what}: non-finite pattern differs"
    fin = np.isfinite(ref)
    excess = np.abs(x[fin] - ref[fin]) - (rtol * np.abs(ref[fin]) + atol)
    k = int(np.argmax(excess))
    assert excess[k] <= 0, (f"{what}: element {np.flatnonzero(fin)[k]} = {x[fin][k]!r} vs "
                            f"{ref[fin][k]!r} (|err| {abs(x[fin][k] - ref[fin][k]):.3e} > "
                            f"{rtol:g}*|ref| + {atol:g})")


def dev_tensor(x, dtype, device="cuda"):
    """Host float array -> CUDA tensor of `dtype` ("f32" or "bf16").  bf16
    values must already be bf16-exact (synth rounds them)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    t = torch.from_numpy(x)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
        # exactness check: the cast must not change any value
        assert torch.equal(t.float(), torch.from_numpy(x)), "input not bf16-exact"
    return t.to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def cu_list(inp: synth.AttnInputs):
    return [int(c) for c in inp.cu_trunk]
