"""Pins for the YaRN tables of the oracle (CPU only).

The pages (NeMo AutoModel ``gpt_oss.rope_utils``, ``RotaryEmbedding`` and
``_compute_concentration_and_inv_freq``; YaRN paper arXiv 2309.00071) print
no numbers, so the pins are the defining properties: plain RoPE at factor 1,
the turn counts that define the two correction dimensions, untouched and
fully interpolated pairs outside them, a linear ramp between them, and the
paper's concentration 0.1 ln s + 1.
"""

import math

import numpy as np
import pytest

from oracle.yarn import (
    concentration_of,
    correction_dim,
    plain_inv_freq,
    rotary_dim_of,
    yarn_inv_freq_and_concentration,
)

GPT = dict(head_dim=64, base=150000.0, factor=32.0, initial_context=4096, ntk_alpha=1.0, ntk_beta=32.0)


def test_factor_one_is_plain_rope_geometric_sequence():
    inv, c = yarn_inv_freq_and_concentration(64, 150000.0, factor=1.0)
    assert c == 1.0
    assert inv.shape == (32,)
    assert inv[0] == 1.0
    # consecutive pairs differ by the constant ratio base^(-2/D)
    ratio = inv[1:] / inv[:-1]
    np.testing.assert_allclose(ratio, math.exp(-2.0 * math.log(150000.0) / 64), rtol=1e-13)
    # last pair: base^(-(D-2)/D)
    assert inv[-1] == pytest.approx(150000.0 ** (-62.0 / 64.0), rel=1e-13)


def test_textbook_value_base10000():
    # RoFormer's theta_i = 10000^(-2(i-1)/d); for d = 128 the second pair is
    # 10000^(-1/64) = 0.8659643233600653 (hand-checked decimal expansion).
    inv = plain_inv_freq(128, 10000.0)
    assert inv[1] == pytest.approx(0.8659643233600653, rel=1e-14)


def test_correction_dims_by_turn_count():
    # d_lo: the pair making ntk_beta turns over L0; d_hi: ntk_alpha turns.
    for turns in (1.0, 32.0):
        d = correction_dim(turns, 64, 150000.0, 4096)
        freq = math.exp(-2.0 * d / 64 * math.log(150000.0))
        assert 4096 * freq / (2 * math.pi) == pytest.approx(turns, rel=1e-12)
    assert correction_dim(32.0, 64, 150000.0, 4096) == pytest.approx(8.0928, abs=1e-4)
    assert correction_dim(1.0, 64, 150000.0, 4096) == pytest.approx(17.3980, abs=1e-4)


def test_concentration_closed_form():
    assert concentration_of(32.0) == pytest.approx(1.3465735902799727, rel=1e-15)
    assert concentration_of(1.0) == 1.0
    assert concentration_of(0.5) == 1.0
    _, c = yarn_inv_freq_and_concentration(**GPT)
    assert c == pytest.approx(1 + 0.1 * math.log(32.0), rel=1e-15)


@pytest.mark.parametrize("ramp", ["index", "paper"])
def test_extrapolated_and_interpolated_pairs(ramp):
    inv, _ = yarn_inv_freq_and_concentration(**GPT, ramp=ramp)
    f = plain_inv_freq(64, 150000.0)
    # more than 32 turns inside 4096 tokens: kept (pairs 0..8)
    np.testing.assert_array_equal(inv[:9], f[:9])
    # fewer than 1 turn: divided by the factor (pairs 18..31)
    np.testing.assert_allclose(inv[18:], f[18:] / 32.0, rtol=1e-15)
    # in between: strictly between the two, decreasing
    assert np.all(inv[9:18] < f[9:18]) and np.all(inv[9:18] > f[9:18] / 32.0)
    assert np.all(np.diff(inv) < 0)


def test_index_ramp_is_linear_in_pair_index():
    inv, _ = yarn_inv_freq_and_concentration(**GPT, ramp="index")
    f = plain_inv_freq(64, 150000.0)
    gamma = (1.0 - inv / f) / (1.0 - 1.0 / 32.0)
    d_lo = correction_dim(32.0, 64, 150000.0, 4096)
    d_hi = correction_dim(1.0, 64, 150000.0, 4096)
    i = np.arange(9, 18)
    np.testing.assert_allclose(gamma[9:18], (i - d_lo) / (d_hi - d_lo), atol=1e-13)
    # spot values quoted for the adopted reading
    assert inv[9] == pytest.approx(3.17057e-2, rel=1e-5)
    assert inv[17] == pytest.approx(1.29319e-4, rel=1e-5)
    assert inv[12] == pytest.approx(6.795e-3, rel=1e-3)


def test_paper_ramp_is_linear_in_turns():
    inv, _ = yarn_inv_freq_and_concentration(**GPT, ramp="paper")
    f = plain_inv_freq(64, 150000.0)
    turns = 4096 * f / (2 * math.pi)
    keep = (inv - f / 32.0) / (f - f / 32.0)
    sel = (turns > 1.0) & (turns < 32.0)
    np.testing.assert_allclose(keep[sel], (turns[sel] - 1.0) / 31.0, atol=1e-13)
    assert inv[12] == pytest.approx(2.673e-3, rel=1e-3)


def test_partial_rotary_uses_rotary_dim():
    assert rotary_dim_of(64, 0.5) == 32
    inv, _ = yarn_inv_freq_and_concentration(64, 150000.0, partial_rotary_factor=0.5)
    assert inv.shape == (16,)
    np.testing.assert_allclose(inv[1] / inv[0], 150000.0 ** (-2.0 / 32.0), rtol=1e-13)
