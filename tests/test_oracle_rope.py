"""Pins for the oracle's RoPE (CPU only).

Rule (NeMo AutoModel ``gpt_oss.rope_utils`` page, ``apply_rotary_emb`` and
``apply_rotary_emb_qk``): half-split pairs (i, i + R), tables carrying the
concentration, features past rotary_dim passed through.  Pins: a worked
example derived by hand (``tests/golden/rope_worked_example.txt``), norm
preservation up to the concentration, dependence of q.k on the relative
position only (also near position 131071), the identity at position 0, the
pairing, and agreement with the complex-multiply formulation.
"""

import os

import numpy as np
import pytest

from oracle.brute import rope_complex
from oracle.rope import default_positions_thd, rope
from oracle.yarn import yarn_inv_freq_and_concentration

HERE = os.path.dirname(__file__)
INV, CONC = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _golden():
    rows = {}
    with open(os.path.join(HERE, "golden", "rope_worked_example.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            key, *vals = line.split()
            rows[key] = np.array([float(v) for v in vals])
    return rows


def test_worked_example():
    g = _golden()
    x = g["x"].reshape(1, 4)
    for c, key in ((1.0, "c1"), (2.0, "c2")):
        out = rope(x, np.array(g["position"][0]), g["inv_freq"], c)
        np.testing.assert_allclose(out[0], g[key], rtol=0, atol=1e-15)


def test_norm_preserved_up_to_concentration():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 7, 64))
    pos = rng.integers(0, 131072, size=5)
    out = rope(x, pos, INV, CONC)
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), CONC * np.linalg.norm(x, axis=-1), rtol=1e-13)


@pytest.mark.parametrize("m,n", [(5, 3), (1000, 17), (131071, 131000), (131071, 0)])
def test_dot_depends_on_relative_position_only(m, n):
    rng = np.random.default_rng(m + n)
    q = rng.standard_normal((1, 64))
    k = rng.standard_normal((1, 64))
    base = float((rope(q, np.array(m), INV, CONC) * rope(k, np.array(n), INV, CONC)).sum())
    for t in (-n, 1, 977, 12345):
        sh = float((rope(q, np.array(m + t), INV, CONC) * rope(k, np.array(n + t), INV, CONC)).sum())
        assert sh == pytest.approx(base, rel=1e-9, abs=1e-9)


def test_position_zero_is_concentration_times_identity():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 3, 64))
    np.testing.assert_array_equal(rope(x, np.zeros(4, np.int64), INV, CONC), CONC * x)


def test_half_split_pairing():
    # a unit vector on feature i moves only into feature i + 32
    for i in (0, 9, 31):
        e = np.zeros((1, 64))
        e[0, i] = 1.0
        out = rope(e, np.array(77), INV, 1.0)[0]
        th = 77 * INV[i]
        expect = np.zeros(64)
        expect[i] = np.cos(th)
        expect[i + 32] = np.sin(th)
        np.testing.assert_allclose(out, expect, atol=1e-15)


def test_agrees_with_complex_formulation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 2, 64))
    pos = np.array([0, 1, 2, 4095, 65536, 131071])
    out = rope(x, pos, INV, CONC)
    for t in range(6):
        for h in range(2):
            ref = rope_complex(list(x[t, h]), int(pos[t]), list(INV), CONC)
            np.testing.assert_allclose(out[t, h], ref, rtol=1e-12, atol=1e-12)


def test_partial_rotary_passthrough():
    inv, c = yarn_inv_freq_and_concentration(64, 150000.0, partial_rotary_factor=0.5)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, 1, 64))
    out = rope(x, np.array([3, 9]), inv, c)
    np.testing.assert_array_equal(out[..., 32:], x[..., 32:])
    np.testing.assert_allclose(np.linalg.norm(out[..., :32], axis=-1), np.linalg.norm(x[..., :32], axis=-1), rtol=1e-13)


def test_thd_positions_restart():
    pos = default_positions_thd(np.array([0, 3, 3, 8]))
    np.testing.assert_array_equal(pos, [0, 1, 2, 0, 1, 2, 3, 4])
