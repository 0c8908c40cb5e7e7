"""Pins of oracle/projection.py (the q, k, v projections with RoPE) to facts
that do not come from its own formula: one-hot inputs pick out a weight
column plus the bias (PyTorch Linear's y = x W^T + b, orientation and split
into heads), PyTorch's own float64 Linear, position 0 (RoPE is the identity
times the concentration), the norm of every rotated head (scaled by the
concentration exactly), linearity, and v never rotated."""

import numpy as np
import torch

from oracle.projection import linear, qkv_rope
from oracle.yarn import yarn_inv_freq_and_concentration

Hq, Hkv, D, HID = 4, 2, 64, 96
N = (Hq + 2 * Hkv) * D


def _w(seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((N, HID)) * 0.05, rng.standard_normal(N) * 0.1


def _tabs():
    return yarn_inv_freq_and_concentration(D, 150000.0, 32.0, 4096, 1.0, 32.0)


def test_one_hot_rows_pick_weight_columns_and_heads():
    w, b = _w(1)
    T = 5
    cols = [0, 7, 33, 64, 95]
    x = np.zeros((T, HID))
    x[np.arange(T), cols] = 1.0
    q, k, v = qkv_rope(x, w, b, np.zeros(T, np.int64), Hq, Hkv, D, rope_tables=None)
    for t, c in enumerate(cols):
        for h in range(Hq):
            for d in (0, 17, 63):
                assert q[t, h, d] == w[h * D + d, c] + b[h * D + d]
        for h in range(Hkv):
            for d in (1, 40):
                assert k[t, h, d] == w[(Hq + h) * D + d, c] + b[(Hq + h) * D + d]
                assert v[t, h, d] == w[(Hq + Hkv + h) * D + d, c] + b[(Hq + Hkv + h) * D + d]


def test_linear_matches_torch_float64():
    w, b = _w(2)
    x = np.random.default_rng(3).standard_normal((7, HID))
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(linear(x, w, b), ref, rtol=1e-13, atol=1e-13)


def test_position_zero_scales_by_concentration():
    w, b = _w(4)
    x = np.random.default_rng(5).standard_normal((3, HID))
    inv_freq, c = _tabs()
    q, k, v = qkv_rope(x, w, b, np.zeros(3, np.int64), Hq, Hkv, D, rope_tables=(inv_freq, c))
    q0, k0, v0 = qkv_rope(x, w, b, np.zeros(3, np.int64), Hq, Hkv, D, rope_tables=None)
    np.testing.assert_allclose(q, c * q0, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(k, c * k0, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(v, v0)


def test_rotation_keeps_head_norms_and_leaves_v():
    w, b = _w(6)
    T = 9
    x = np.random.default_rng(7).standard_normal((T, HID))
    pos = np.array([0, 1, 5, 100, 4095, 4096, 70000, 131071, 3])
    inv_freq, c = _tabs()
    q, k, v = qkv_rope(x, w, b, pos, Hq, Hkv, D, rope_tables=(inv_freq, c))
    q0, k0, v0 = qkv_rope(x, w, b, pos, Hq, Hkv, D, rope_tables=None)
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), c * np.linalg.norm(q0, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(k, axis=-1), c * np.linalg.norm(k0, axis=-1), rtol=1e-12)
    np.testing.assert_array_equal(v, v0)


def test_linear_in_x_without_bias():
    w, _ = _w(8)
    rng = np.random.default_rng(9)
    x1, x2 = rng.standard_normal((4, HID)), rng.standard_normal((4, HID))
    np.testing.assert_allclose(linear(2.5 * x1 + x2, w, None), 2.5 * linear(x1, w, None) + linear(x2, w, None),
                               rtol=1e-12, atol=1e-12)
