"""Shared helpers of the GPU parity tests: upload seeded inputs, compare a
kernel's output with the float64 oracle.

Tolerance (bf16 inputs, fp32 accumulation, stated for outputs of unit scale):
every element within 1e-2 of the oracle on the unit scale -- i.e.
|got - ref| <= 1e-2 * max(1, |ref|) -- and mean-abs error <= 1e-3.  The
scale factor only matters above |ref| = 1: a bf16 output of magnitude 2..4 is
quantised in steps of 2^-6, so half a step (7.8e-3) of the 1e-2 budget is
spent by the output format alone, and above 4 the step itself exceeds 1e-2.
"""

from __future__ import annotations

import numpy as np
import torch

from attention_yarn_rope_b200.workloads import to_torch_bf16

MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def dev(x, device="cuda:0"):
    return to_torch_bf16(x, device)


def f32(x: np.ndarray, device="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(device)


def i32(x, device="cuda:0"):
    return torch.as_tensor(np.asarray(x, np.int32), device=device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_parity(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    scaled = err / np.maximum(1.0, np.abs(ref))
    mx, mean, smx = float(err.max()), float(err.mean()), float(scaled.max())
    assert smx <= max_abs, f"{what}: scaled max error {smx:.3e} > {max_abs} (max-abs {mx:.3e}, mean {mean:.3e})"
    assert mean <= mean_abs, f"{what}: mean-abs {mean:.3e} > {mean_abs}"
    return mx, mean


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significand bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)
