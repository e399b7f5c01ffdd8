"""Shared helpers of the GPU parity tests: moving seeded inputs to the device
and the tolerance gates.

Gates (fixed by the spec of the path; readings stated in the design notes):

* float32: max|err| <= 1e-4 * max|ref| over the output tensor.
* bfloat16: "2e-2 absolute on unit-scale outputs", held on every element
  for the computation, plus the output's own final rounding:
  |err| <= 2e-2 * min(1, RMS(ref_row)) + ulp_bf16(ref) / 2, where a row is
  the last axis (the head_dim-vector of one head at one token, or a token's
  hidden vector).  On a row of unit (or larger) scale the first term is the
  spec's 2e-2 absolute; on a smaller row it is 2% of the row's own scale
  (decode outputs, RMS ~0.05, are held to ~1e-3).  The second term is half
  the spacing of bf16 values at the reference (2^-8 of |ref| at most): no
  bf16 output can be closer than that to a reference midway between two
  bf16 values, so without it an element above 8 in magnitude (spacing
  0.0625) could never pass even when correctly rounded.
  ``col_scale`` names channels that the inputs scaled on purpose (the
  long-context workload multiplies 0.1% of V's channels by 20); attention
  is linear in V, so such an output channel is that factor times a
  unit-scale output, and its row RMS and its bound are taken on that scale.
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


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    """Half the spacing of bfloat16 values (8 significant bits) at |ref|:
    2^(floor(log2|ref|) - 8); 0 at 0."""
    a = np.abs(np.asarray(ref, dtype=np.float64))
    _, e = np.frexp(a)                      # a = m * 2**e, 0.5 <= m < 1
    return np.where(a > 0, np.ldexp(1.0, e - 9), 0.0)


def gate(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "", col_scale=None):
    """Assert the spec's tolerance; rows are the last axis.  ``col_scale``
    (broadcastable to ``ref``) is the factor by which the inputs scaled an
    output channel on purpose (1 elsewhere)."""
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
    scale = np.ones_like(ref) if col_scale is None else np.broadcast_to(np.asarray(col_scale, np.float64), ref.shape)
    unit = ref / scale
    rms = np.sqrt(np.mean(unit * unit, axis=-1, keepdims=True))
    lim = BF16_TOL * scale * np.minimum(1.0, rms) + half_ulp_bf16(ref)
    over = err > lim
    if np.any(over):
        ratio = np.where(lim > 0, err / np.where(lim > 0, lim, 1.0), np.inf)
        idx = np.unravel_index(np.argmax(np.where(over, ratio, -1.0)), ratio.shape)
        raise AssertionError(f"{what}: err {err[idx]:.3e} at {idx} exceeds 2e-2 x min(1, row RMS) + ulp/2 = {lim[idx]:.3e} "
                             f"(row RMS {float(rms[idx[:-1]][0]):.3e}, ref {ref[idx]:.4f}, got {got[idx]:.4f})")
    ok = lim > 0
    return float((err[ok] / lim[ok]).max()) if np.any(ok) else 0.0
