"""Rotary position embedding of q and k, float64.

Source: NeMo AutoModel ``gpt_oss.rope_utils`` page:

* ``apply_rotary_emb(x, cos, sin)``: cos/sin carry ``rotary_dim // 2``
  entries; the first ``rotary_dim`` features of x are rotated and the rest
  pass through unchanged.
* ``apply_rotary_emb_qk(q, k, freqs_cis, format, ..., concentration)``: q and
  k are rotated with the same tables; the tables carry the concentration
  ("cosine/sine tables with concentration applied"; for the fused path "scale
  applied after TE fused RoPE").  The fused form receives "duplicated
  angles" over the two halves of rotary_dim, which fixes the pairing as
  half-split: feature i is paired with feature i + R, R = rotary_dim / 2.

For pair i of a token at position p, theta = p * inv_freq[i], and

    x'_i     = c * (x_i cos theta - x_{i+R} sin theta)
    x'_{i+R} = c * (x_{i+R} cos theta + x_i sin theta)

with c the concentration.  No table is rounded to a lower precision.
"""

from __future__ import annotations

import numpy as np


def rope(x: np.ndarray, positions: np.ndarray, inv_freq: np.ndarray, concentration: float) -> np.ndarray:
    """Rotate ``x[..., H, D]`` at ``positions[...]`` (broadcast over H).

    ``inv_freq`` has R = rotary_dim/2 entries; features ``[2R, D)`` pass
    through unchanged (partial rotary).
    """
    x = np.asarray(x, dtype=np.float64)
    R = inv_freq.shape[0]
    D = x.shape[-1]
    if 2 * R > D:
        raise ValueError("rotary_dim exceeds head_dim")
    pos = np.asarray(positions, dtype=np.float64)
    theta = pos[..., None] * inv_freq  # [..., R]
    cos = np.cos(theta)[..., None, :]  # broadcast over heads
    sin = np.sin(theta)[..., None, :]
    lo = x[..., :R]
    hi = x[..., R:2 * R]
    out = x.copy()
    out[..., :R] = concentration * (lo * cos - hi * sin)
    out[..., R:2 * R] = concentration * (hi * cos + lo * sin)
    if 2 * R < D:
        out[..., 2 * R:] = x[..., 2 * R:]
    return out


def default_positions_bshd(B: int, S: int) -> np.ndarray:
    """BSHD default positions 0..S-1 for every batch row."""
    return np.broadcast_to(np.arange(S, dtype=np.int64), (B, S)).copy()


def default_positions_thd(cu_seqlens: np.ndarray) -> np.ndarray:
    """Packed THD default positions: restart at 0 at every sequence start."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    pos = np.empty(T, dtype=np.int64)
    for s in range(len(cu) - 1):
        pos[cu[s]:cu[s + 1]] = np.arange(cu[s + 1] - cu[s])
    return pos
