"""Attention over key blocks and the log-sum-exp merge (test infrastructure only).

Context parallelism for the full-context layers (the ``cp_size`` /
``cp_rank`` arguments of ``apply_rotary_emb_qk`` on the NeMo AutoModel
gpt_oss.rope_utils page) computes each query shard's attention one key
shard at a time and merges the pieces.  The pages give no formula for the
merge; it follows from the definition in :mod:`oracle.attention`: with the
visible keys of row i split into disjoint blocks b,

    Z_i = exp(sink_h) + sum_b sum_{j in b} exp(s_ij)
        = exp(sink_h) + sum_b exp(lse_ib),   lse_ib = log sum_{j in b} exp(s_ij)
    o_i = sum_b exp(lse_ib) o_ib / Z_i,      o_ib = sum_{j in b} exp(s_ij - lse_ib) v_j

so each block returns its own normalised output and log-sum-exp, with no
sink (a block with no visible key returns lse = -inf), and the sink enters
once, in the merge.  Blocks are given by global token indices, so the causal
mask and the window apply across them; RoPE takes the global positions.
"""

from __future__ import annotations

import numpy as np

from .attention import _visible_mask


def block_attention(q_rot, k_rot, v, scale, window, q_off: int, k_off: int):
    """One block: queries ``q_rot [Lq, Hq, D]`` at global rows q_off.., keys
    ``k_rot / v [Lk, Hkv, D]`` at global rows k_off.. (both already rotated).
    Returns ``(o [Lq, Hq, D], lse [Hq, Lq])`` over the visible pairs of the
    block, no sink; rows that see no key of the block get o = 0, lse = -inf."""
    q_rot = np.asarray(q_rot, np.float64)
    k_rot = np.asarray(k_rot, np.float64)
    v = np.asarray(v, np.float64)
    Lq, Hq, D = q_rot.shape
    Lk, Hkv = k_rot.shape[:2]
    G = Hq // Hkv
    vis = _visible_mask(np.arange(q_off, q_off + Lq), np.arange(k_off, k_off + Lk), window)
    o = np.zeros((Lq, Hq, D))
    lse = np.full((Hq, Lq), -np.inf)
    rows = vis.any(axis=1)
    for h in range(Hq):
        g = h // G
        s = scale * (q_rot[:, h, :] @ k_rot[:, g, :].T)
        s = np.where(vis, s, -np.inf)
        m = np.where(rows, s.max(axis=1), 0.0)
        e = np.exp(s - m[:, None])
        z = e.sum(axis=1)
        o[rows, h, :] = (e[rows] @ v[:, g, :]) / z[rows, None]
        lse[h, rows] = m[rows] + np.log(z[rows])
    return o, lse


def merge_blocks(parts, sinks):
    """Merge block results ``[(o_b [L, Hq, D], lse_b [Hq, L]), ...]`` of the same
    query rows and fold the sink in once: ``(o [L, Hq, D], lse [Hq, L])`` of
    the sink attention over the union of the blocks' keys."""
    sinks = np.asarray(sinks, np.float64)
    lses = np.stack([p[1] for p in parts])                     # [nb, Hq, L]
    m = np.maximum(lses.max(axis=0), sinks[:, None])           # [Hq, L]
    w = np.exp(lses - m[None])                                 # exp(lse_b - m), 0 for -inf
    z = np.exp(sinks[:, None] - m) + w.sum(axis=0)
    o = sum(np.transpose(wb, (1, 0))[:, :, None] * p[0] for wb, p in zip(w, parts))
    return o / np.transpose(z, (1, 0))[:, :, None], m + np.log(z)
