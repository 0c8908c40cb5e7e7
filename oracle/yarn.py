"""YaRN rotary frequencies and attention concentration, float64.

Source: NeMo AutoModel, ``nemo_automodel.components.models.gpt_oss.rope_utils``
page, class ``RotaryEmbedding(head_dim, base, dtype, initial_context_length=4096,
scaling_factor=1.0, ntk_alpha=1.0, ntk_beta=32.0, partial_rotary_factor=1.0)``,
attribute ``rotary_dim = int(head_dim * partial_rotary_factor)`` and method
``_compute_concentration_and_inv_freq`` ("See YaRN paper", arXiv 2309.00071;
"uses rotary_dim instead of head_dim").  The concentration is the
``yarn_concentration = yarn_get_mscale(rope_scaling['factor'])`` attribute of
``GptOssAttention`` on the ``gpt_oss.layers`` page.

The pages name the parameters but print no formula; the YaRN paper supplies
the mathematics ("NTK-by-parts" interpolation, Sec. 3.2, and the attention
temperature, Sec. 3.4):

* plain RoPE frequencies  f_i = base ** (-2 i / rotary_dim),  i in [0, R),
  R = rotary_dim / 2;
* a pair whose wavelength 2 pi / f_i is short compared with the original
  context L0 (more than ``ntk_beta`` turns inside L0) is extrapolated, i.e.
  kept at f_i; a pair with fewer than ``ntk_alpha`` turns inside L0 is
  interpolated, f_i / factor; pairs in between are blended;
* the concentration (the paper's sqrt(1/t)) is 0.1 ln(factor) + 1, and
  multiplies both rotated q and rotated k.

Reading of the blend (the pages leave it open): ``ramp="index"`` ramps
linearly in the pair index i between the two (unrounded) correction
dimensions d_lo and d_hi at which a pair makes exactly ntk_beta and
ntk_alpha turns inside L0; ``ramp="paper"`` ramps linearly in the number of
turns r = L0 f_i / (2 pi), the YaRN paper's gamma(r).  Both agree outside
(d_lo, d_hi).  "index" is the adopted reading.
"""

from __future__ import annotations

import math

import numpy as np


def rotary_dim_of(head_dim: int, partial_rotary_factor: float = 1.0) -> int:
    """``rotary_dim = int(head_dim * partial_rotary_factor)`` (rope_utils page)."""
    return int(head_dim * partial_rotary_factor)


def plain_inv_freq(rotary_dim: int, base: float) -> np.ndarray:
    """Textbook RoPE inverse frequencies base^(-2i/rotary_dim), i in [0, R)."""
    if rotary_dim % 2:
        raise ValueError("rotary_dim must be even")
    i = np.arange(rotary_dim // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * i / rotary_dim)


def correction_dim(turns: float, rotary_dim: int, base: float, initial_context: int) -> float:
    """Real pair index d at which the pair makes ``turns`` full turns over the
    original context L0, i.e. L0 * base^(-2d/rotary_dim) / (2 pi) == turns."""
    return (rotary_dim / 2.0) * math.log(initial_context / (turns * 2.0 * math.pi)) / math.log(base)


def concentration_of(factor: float) -> float:
    """YaRN attention concentration (paper Sec. 3.4): 0.1 ln(s) + 1 for s > 1, else 1."""
    if factor <= 1.0:
        return 1.0
    return 0.1 * math.log(factor) + 1.0


def yarn_inv_freq_and_concentration(
    head_dim: int,
    base: float,
    factor: float = 1.0,
    initial_context: int = 4096,
    ntk_alpha: float = 1.0,
    ntk_beta: float = 32.0,
    partial_rotary_factor: float = 1.0,
    ramp: str = "index",
):
    """Return ``(inv_freq[R] float64, concentration float)``.

    ``factor <= 1`` gives plain RoPE and concentration 1.
    """
    rdim = rotary_dim_of(head_dim, partial_rotary_factor)
    f = plain_inv_freq(rdim, base)
    if factor <= 1.0:
        return f, 1.0
    conc = concentration_of(factor)
    if ramp == "index":
        d_lo = correction_dim(ntk_beta, rdim, base, initial_context)
        d_hi = correction_dim(ntk_alpha, rdim, base, initial_context)
        i = np.arange(rdim // 2, dtype=np.float64)
        gamma = np.clip((i - d_lo) / (d_hi - d_lo), 0.0, 1.0)  # 0: keep, 1: divide by factor
    elif ramp == "paper":
        turns = initial_context * f / (2.0 * math.pi)
        keep = np.clip((turns - ntk_alpha) / (ntk_beta - ntk_alpha), 0.0, 1.0)
        gamma = 1.0 - keep
    else:
        raise ValueError(f"unknown ramp reading {ramp!r}")
    inv_freq = f * (1.0 - gamma) + (f / factor) * gamma
    return inv_freq, conc
