"""Agreement rules between the CUDA path and the fp64 oracle.

fp32 inputs: every element |g - o| <= 1e-4 * max(1, |o|).
bf16 inputs (fp32 accumulation): max |g - o| <= 2e-2 * max |o| over the
tensor, and every element |g - o| <= 2e-2 * (|o| + rms(o)).
Gradients of the backward pass in fp32 (``grad=True``): max |g - o| <= 1e-4
max |o| and every element |g - o| <= 1e-4 (|o| + rms(o)).
These are the 1e-4 (fp32) and 2e-2 relative (bf16) bounds of the task; the
per-element form for bf16 measures each error against the element's own size
plus the tensor's rms, so near-zero outputs are not held to a relative bound
that rounding of their (cancelling) terms cannot meet.

The tensor-scaled fp32 form is for gradients only, and only when a test asks
for it with ``grad=True``: each gradient element is a sum over a chunk's
tokens and channels whose terms scale with the tensor, not with the element.
Forward outputs, states and decode steps in fp32 always take the element-wise
1e-4 * max(1, |o|) rule, and nothing else in this file widens a bound.
"""
from __future__ import annotations

import numpy as np
import torch

FP32_TOL = 1e-4
BF16_TOL = 2e-2


def _np(a):
    if isinstance(a, torch.Tensor):
        return a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def report(gpu, ref):
    g, o = _np(gpu), _np(ref)
    d = np.abs(g - o)
    i = int(np.argmax(d)) if d.size else 0
    rel = d / np.maximum(np.abs(o), 1e-30)
    rms = float(np.sqrt(np.mean(o * o))) if d.size else 0.0
    # worst element against the bf16 element-wise bound (1.0 = at the bound)
    ratio = d / (BF16_TOL * (np.abs(o) + rms) + 1e-300)
    w = int(np.argmax(ratio)) if d.size else 0
    return {"max_abs": float(d.max()) if d.size else 0.0,
            "max_rel": float(rel.max()) if d.size else 0.0,
            "argmax": np.unravel_index(i, d.shape) if d.size else (),
            "ref_max": float(np.abs(o).max()) if d.size else 0.0,
            "ref_rms": rms, "worst_vs_bf16_bound": float(ratio.max()) if d.size else 0.0,
            "worst_at": np.unravel_index(w, d.shape) if d.size else (),
            "worst_gpu_ref": (float(g.flat[w]), float(o.flat[w])) if d.size else ()}


def assert_close(gpu, ref, dtype, what="", grad=False):
    """``grad`` marks a gradient of the backward pass: for fp32 it is held to
    the scaled form at 1e-4 (max |g - o| <= 1e-4 max |o| and every element
    |g - o| <= 1e-4 (|o| + rms(o))), because each gradient element is a sum
    over a chunk's tokens and channels whose terms scale with the tensor, not
    with the element, so their fp32 rounding does too."""
    g, o = _np(gpu), _np(ref)
    assert g.shape == o.shape, f"{what}: shape {g.shape} != {o.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values in the CUDA result"
    d = np.abs(g - o)
    if d.size == 0:
        return
    if dtype in (torch.float32, "f32") and grad:
        omax = np.abs(o).max()
        rms = float(np.sqrt(np.mean(o * o)))
        assert d.max() <= FP32_TOL * omax + 1e-30, (
            f"{what}: max abs err {d.max():.3e} > 1e-4 * max|o|; {report(g, o)}")
        bad = d > FP32_TOL * (np.abs(o) + rms)
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond 1e-4 * (|o| + rms); "
                               f"{report(g, o)}")
    elif dtype in (torch.float32, "f32"):
        bound = FP32_TOL * np.maximum(1.0, np.abs(o))
        bad = d > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the fp32 bound; "
                               f"{report(g, o)}")
    else:
        omax = np.abs(o).max()
        rms = float(np.sqrt(np.mean(o * o)))
        assert d.max() <= BF16_TOL * omax + 1e-30, (
            f"{what}: max abs err {d.max():.3e} > 2e-2 * max|o| = {BF16_TOL * omax:.3e}; "
            f"{report(g, o)}")
        bad = d > BF16_TOL * (np.abs(o) + rms)
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond 2e-2 * (|o| + rms); "
                               f"{report(g, o)}")
