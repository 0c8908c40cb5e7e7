"""Shared helpers of the GPU parity tests: upload seeded inputs, compare a
kernel's output with the float64 oracle.

Bar (bf16 inputs, fp32 accumulation; max-abs 1e-2 and mean-abs 1e-3 on
outputs of unit scale):

* bf16 outputs (``assert_parity``): every element with |ref| <= 4 within
  1e-2 of the oracle, raw.  Above 4 the bf16 format alone rounds by up to
  half a spacing (2^-6 = 1.56e-2 for |o| in [4, 8)), more than the whole bar,
  so there an element may differ by 1e-2 plus half the bf16 spacing at
  |ref|.  Mean-abs error <= 1e-3 over all elements.
* fp32 log-sum-exp (``assert_lse_parity``): every element within 1e-2 of
  the oracle, raw, and mean-abs <= 1e-3: lse is written in fp32, so no format
  allowance applies.

Each failure message prints the raw max-abs error, where it occurred and the
mean.
"""

from __future__ import annotations

import numpy as np
import torch

from attention_yarn_rope_b200.workloads import to_torch_bf16

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-2
BF16_ALLOWANCE_ABOVE = 4.0


def dev(x, device="cuda:0"):
    return to_torch_bf16(x, device)


def f32(x: np.ndarray, device="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(device)


def i32(x, device="cuda:0"):
    return torch.as_tensor(np.asarray(x, np.int32), device=device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def out_bar(ref: np.ndarray, max_abs=MAX_ABS) -> np.ndarray:
    """Per-element bar of a bf16 output: max_abs where |ref| <= 4, plus half
    the bf16 spacing at |ref| above 4 (the output format's own rounding)."""
    a = np.abs(np.asarray(ref, np.float64))
    return np.where(a <= BF16_ALLOWANCE_ABOVE, max_abs, max_abs + 0.5 * bf16_ulp(a))


def _report(what, err, ref, mean):
    i = int(np.argmax(err))
    return (f"{what}: raw max-abs {float(err.flat[i]):.3e} at |ref| = {abs(float(ref.flat[i])):.3f} "
            f"(flat index {i}), mean-abs {mean:.3e}")


def assert_parity(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    """bf16 output against the oracle: raw 1e-2 where |ref| <= 4 (plus half a
    bf16 spacing above 4), mean-abs 1e-3."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mean = float(err.mean()) if err.size else 0.0
    if err.size:
        bad = err > out_bar(ref, max_abs)
        assert not bad.any(), f"{int(bad.sum())} elements over the bar; " + _report(what, err, ref, mean)
    assert mean <= mean_abs, _report(what, err, ref, mean)
    return (float(err.max()) if err.size else 0.0), mean


def assert_lse_parity(got: np.ndarray, ref: np.ndarray, what: str, max_abs=LSE_MAX_ABS, mean_abs=MEAN_ABS):
    """fp32 log-sum-exp against the oracle: raw max-abs and mean-abs."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite lse"
    err = np.abs(got - ref)
    mean = float(err.mean()) if err.size else 0.0
    if err.size:
        assert float(err.max()) <= max_abs, _report(what, err, ref, mean)
    assert mean <= mean_abs, _report(what, err, ref, mean)
    return (float(err.max()) if err.size else 0.0), mean


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significand bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)
