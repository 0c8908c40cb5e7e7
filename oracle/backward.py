"""Gradients of the sink attention with RoPE, float64 (test infrastructure only).

The pages define the forward pass (``oracle.attention``: NeMo AutoModel
``gpt_oss.layers`` page, ``GptOssAttention``; ``gpt_oss.rope_utils`` page,
``apply_rotary_emb_qk``) and describe training the model with NeMo AutoModel,
which needs its gradients; they print no backward formula.  This module is the
exact derivative of that forward definition, written out by the chain rule
for the scalar ``L = sum(dout * out)``:

For one sequence, query head h (kv head g), with the forward's weights
``w_ij`` (visible pairs only) and sink share ``a_i = exp(sink_h - lse_i)``:

    dv_j[g]   += sum_i w_ij dout_i[h]
    dP_ij      = <dout_i[h], v_j[g]>
    D_i        = sum_j w_ij dP_ij  (= <dout_i[h], o_i[h]>; formed from a
                                      stored output when one is given)
    dS_ij      = w_ij (dP_ij - D_i)
    dsink_h   += -sum_i a_i D_i          (the sink column has no value row)
    dq'_i[h]   = scale * sum_j dS_ij k'_j[g]
    dk'_j[g]  += scale * sum_i dS_ij q'_i[h]

and through RoPE, which is linear (``x' = c R(theta) x`` per pair), the raw
gradients are ``dq = c R(theta)^T dq'`` and ``dk = c R(theta)^T dk'``
(:func:`rope_transpose`).  The weights are recomputed here from the
definition; as in the forward oracle, rows go in blocks, each evaluated over
the keys it can see, and nothing else is tiled or reordered.
"""

from __future__ import annotations

import numpy as np

from .attention import _ROW_BLOCK, _visible_mask
from .rope import default_positions_bshd, default_positions_thd, rope


def rope_transpose(g: np.ndarray, positions: np.ndarray, inv_freq: np.ndarray, concentration: float) -> np.ndarray:
    """Apply ``c R(theta)^T`` to ``g[..., H, D]``: the adjoint of :func:`oracle.rope.rope`.

    For pair i, ``(x, y) -> c (x cos + y sin, y cos - x sin)``; features past
    the rotary dimension pass through."""
    g = np.asarray(g, dtype=np.float64)
    R = inv_freq.shape[0]
    theta = np.asarray(positions, dtype=np.float64)[..., None] * inv_freq
    cos = np.cos(theta)[..., None, :]
    sin = np.sin(theta)[..., None, :]
    x = g[..., :R]
    y = g[..., R:2 * R]
    out = g.copy()
    out[..., :R] = concentration * (x * cos + y * sin)
    out[..., R:2 * R] = concentration * (y * cos - x * sin)
    return out


def sink_attention_sequence_bwd(q_rot, k_rot, v, sinks, scale, window, dout, out=None):
    """One sequence.  q_rot / dout ``[L, Hq, D]``, k_rot / v ``[L, Hkv, D]``.
    Returns ``dq_rot [L, Hq, D]``, ``dk_rot [L, Hkv, D]``, ``dv [L, Hkv, D]``,
    ``dsink [Hq]``.  ``out`` (``[L, Hq, D]``), when given, is the forward
    output as the caller stores it, and ``D_i = <dout_i, out_i>`` is formed
    from it (with the exact output this is the same number as
    ``sum_j w_ij dP_ij``); otherwise D comes from the exact weights.  Rows are
    taken in blocks of the forward's size, each over the key range it can see
    (masked pairs contribute nothing); the key-side gradients add up over the
    blocks."""
    q_rot = np.asarray(q_rot, np.float64)
    k_rot = np.asarray(k_rot, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    sinks = np.asarray(sinks, np.float64)
    if out is not None:
        out = np.asarray(out, np.float64)
    L, Hq, D = q_rot.shape
    Hkv = k_rot.shape[1]
    G = Hq // Hkv
    dq = np.zeros_like(q_rot)
    dk = np.zeros_like(k_rot)
    dv = np.zeros_like(v)
    dsink = np.zeros(Hq, np.float64)
    for r0 in range(0, L, _ROW_BLOCK):
        r1 = min(L, r0 + _ROW_BLOCK)
        k0 = max(0, r0 - window + 1) if window > 0 else 0
        vis = _visible_mask(np.arange(r0, r1), np.arange(k0, r1), window)
        for h in range(Hq):
            g = h // G
            s = scale * (q_rot[r0:r1, h, :] @ k_rot[k0:r1, g, :].T)
            s = np.where(vis, s, -np.inf)
            m = np.maximum(sinks[h], s.max(axis=1))
            e = np.exp(s - m[:, None])
            z = np.exp(sinks[h] - m) + e.sum(axis=1)
            w = e / z[:, None]                       # weights of the visible pairs
            share = np.exp(sinks[h] - m) / z         # the sink's share a_i
            dv[k0:r1, g, :] += w.T @ dout[r0:r1, h, :]
            dP = dout[r0:r1, h, :] @ v[k0:r1, g, :].T
            if out is None:
                Drow = (w * dP).sum(axis=1)
            else:
                Drow = (dout[r0:r1, h, :] * out[r0:r1, h, :]).sum(axis=1)
            dS = w * (dP - Drow[:, None])
            dsink[h] -= (share * Drow).sum()
            dq[r0:r1, h, :] = scale * (dS @ k_rot[k0:r1, g, :])
            dk[k0:r1, g, :] += scale * (dS.T @ q_rot[r0:r1, h, :])
    return dq, dk, dv, dsink


def _grads_of_sequence(q, k, v, sinks, scale, window, dout, pos, rope_tables, out):
    if rope_tables is None:
        dq, dk, dv, ds = sink_attention_sequence_bwd(q, k, v, sinks, scale, window, dout, out)
        return dq, dk, dv, ds
    inv_freq, conc = rope_tables
    qr = rope(q, pos, inv_freq, conc)
    kr = rope(k, pos, inv_freq, conc)
    dqr, dkr, dv, ds = sink_attention_sequence_bwd(qr, kr, v, sinks, scale, window, dout, out)
    return rope_transpose(dqr, pos, inv_freq, conc), rope_transpose(dkr, pos, inv_freq, conc), dv, ds


def attn_bwd_bshd(q, k, v, sinks, scale, window, dout, rope_tables=None, positions=None, out=None):
    """Gradients of ``sum(dout * attn_fwd_bshd(q, k, v, ...).out)``: ``dq [B, S,
    Hq, D]``, ``dk``, ``dv [B, S, Hkv, D]``, ``dsinks [Hq]`` (summed over the
    batch).  ``rope_tables`` and ``positions`` as for the forward; ``out``
    optional, the stored forward output D is formed from."""
    B, S = q.shape[:2]
    if positions is None:
        positions = default_positions_bshd(B, S)
    dq = np.zeros(q.shape, np.float64)
    dk = np.zeros(k.shape, np.float64)
    dv = np.zeros(v.shape, np.float64)
    dsinks = np.zeros(q.shape[2], np.float64)
    for b in range(B):
        dq[b], dk[b], dv[b], ds = _grads_of_sequence(q[b], k[b], v[b], sinks, scale, window, dout[b], positions[b],
                                                     rope_tables, None if out is None else out[b])
        dsinks += ds
    return dq, dk, dv, dsinks


def attn_bwd_thd(q, k, v, sinks, cu_seqlens, scale, window, dout, rope_tables=None, positions=None, out=None):
    """Packed THD gradients: ``dq [T, Hq, D]``, ``dk``, ``dv [T, Hkv, D]``,
    ``dsinks [Hq]`` (summed over the sequences); ``out`` as for
    :func:`attn_bwd_bshd`."""
    cu = np.asarray(cu_seqlens, np.int64)
    if positions is None:
        positions = default_positions_thd(cu)
    dq = np.zeros(q.shape, np.float64)
    dk = np.zeros(k.shape, np.float64)
    dv = np.zeros(v.shape, np.float64)
    dsinks = np.zeros(q.shape[1], np.float64)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        dq[a:b], dk[a:b], dv[a:b], ds = _grads_of_sequence(q[a:b], k[a:b], v[a:b], sinks, scale, window, dout[a:b],
                                                           positions[a:b], rope_tables,
                                                           None if out is None else out[a:b])
        dsinks += ds
    return dq, dk, dv, dsinks
