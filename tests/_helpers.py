"""Shared helpers of the GPU parity tests: moving seeded inputs to the device
and the tolerance gates.

Gates (fixed by the spec of the path; readings stated in the design notes):

* float32: max|err| <= 1e-4 * max|ref| over the output tensor.
* bfloat16: "2e-2 absolute on unit-scale outputs".  The scale of an output is
  taken per output row (the head_dim-vector of one head at one token) as its
  RMS, and an element larger than that scale is held to 2e-2 of itself (no
  bf16 value is closer than 2^-8 relative to its reference):
  |err| <= 2e-2 * max(RMS(ref_row), |ref|).  On a unit-scale row with
  elements up to 1 this is exactly 2e-2 absolute; decode outputs (RMS ~0.05)
  are held to ~1e-3.  Where V has outlier channels (x20 in the long-context
  workload) an output channel has a scale of its own, so attention outputs
  compared as [rows, hd] also take the RMS of their (head, channel) over the
  compared rows into the max.
* KV-cache layout: bit-exact (integer inputs with exact fp32 sums).
"""
from __future__ import annotations

import numpy as np
import torch

from workloads import Tensor, bf16_to_f32

BF16_TOL = 2e-2
F32_TOL = 1e-4


def dev(t: Tensor, device="cuda") -> torch.Tensor:
    if t.dtype == "bf16":
        return torch.from_numpy(t.store.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(t.store)).to(device)


def dev_i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a device tensor."""
    if t.dtype == torch.bfloat16:
        bits = t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
        with np.errstate(invalid="ignore"):
            return bf16_to_f32(bits).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.detach().cpu().numpy().view(np.uint32)


def gate(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "", heads=None):
    """Assert the spec's tolerance; rows are the last axis.  ``heads`` (one id
    per row of a 2-D ``[rows, hd]`` comparison) groups rows by attention head
    so that each (head, channel) also gets its own RMS scale."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        bound = F32_TOL * max(np.max(np.abs(ref)), 1e-30)
        worst = float(err.max()) if err.size else 0.0
        assert worst <= bound, f"{what}: max|err| {worst:.3e} > {bound:.3e}"
        return worst / bound if bound else 0.0
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    scale = np.maximum(rms, np.abs(ref))
    if heads is not None:
        heads = np.asarray(heads)
        col = np.zeros_like(ref)
        for hid in np.unique(heads):
            sel = heads == hid
            col[sel] = np.sqrt(np.mean(ref[sel] ** 2, axis=0, keepdims=True))
        scale = np.maximum(scale, col)
    lim = BF16_TOL * np.maximum(scale, 1e-6)
    ratio = err / lim
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        idx = np.unravel_index(np.argmax(ratio), ratio.shape)
        raise AssertionError(f"{what}: err {err[idx]:.3e} at {idx} exceeds 2e-2 x row RMS "
                             f"{float(rms[idx[:-1]][0]):.3e} (ref {ref[idx]:.4f}, got {got[idx]:.4f})")
    return worst
