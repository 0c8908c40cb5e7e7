"""Grouped-query causal softmax attention with a per-head sink, float64.

Sources:
* NeMo AutoModel ``gpt_oss.layers`` page, ``GptOssAttention``: attributes
  ``sinks``, ``sliding_window``, ``softmax_scale = head_dim ** -0.5``,
  ``num_attention_heads``, ``num_key_value_heads``; ``_has_thd_metadata``
  (packed THD inputs carry ``cu_seqlens``).
* Transformers v4.55.0 release notes, "Architecture": layers alternate
  between full context and a sliding 128-token window; "a learned attention
  sink per-head, where the denominator of the softmax has an additional
  additive value".
* NeMo AutoModel ``gpt_oss.model`` page, ``GptOssForCausalLM.forward``: BSHD
  ``[B, S]`` or packed THD ``[1, T]`` inputs with ``cu_seqlens`` in
  ``attn_kwargs``.
* gpt-oss-20b module tree (blog page "gpt-oss-20b 模型结构"): q_proj
  2880 -> 4096 = 64 heads x 64, k_proj / v_proj 2880 -> 512 = 8 heads x 64.

Definition computed (for one sequence, query row i, q-head h, kv-head
g = h // (Hq / Hkv), scale = softmax_scale):

    s_ij   = scale * <q'_i[h], k'_j[g]>            (q', k' after RoPE)
    visible(i, j) = j <= i  and  (window == 0  or  i - j < window)
    M_i    = max(sink_h, max_{visible j} s_ij)
    Z_i    = exp(sink_h - M_i) + sum_{visible j} exp(s_ij - M_i)
    w_ij   = exp(s_ij - M_i) / Z_i
    o_i[h] = sum_{visible j} w_ij v_j[g]
    lse_i  = M_i + ln Z_i

The sink enters the denominator only; ``sink_h`` is compared in the units of
the scaled logits.  A sink of -inf gives standard softmax attention.
Visibility follows token order inside a sequence; positions feed RoPE only.
Tokens of different packed sequences never see each other.

Masked pairs contribute nothing to the definition, so the code evaluates the
logits only over the key range a row block can see (the band for a sliding
window); nothing else is blocked, fused or reordered.
"""

from __future__ import annotations

import numpy as np

from .rope import default_positions_bshd, default_positions_thd, rope

_ROW_BLOCK = 512


def _visible_mask(rows: np.ndarray, keys: np.ndarray, window: int) -> np.ndarray:
    vis = keys[None, :] <= rows[:, None]
    if window > 0:
        vis &= (rows[:, None] - keys[None, :]) < window
    return vis


def sink_attention_sequence(q_rot, k_rot, v, sinks, scale, window, return_weights=False):
    """One sequence.  q_rot ``[L, Hq, D]``, k_rot / v ``[L, Hkv, D]`` (float64),
    sinks ``[Hq]``.  Returns ``out [L, Hq, D]``, ``lse [Hq, L]`` and, if asked,
    ``(weights [Hq, L, L], sink_share [Hq, L])``."""
    q_rot = np.asarray(q_rot, np.float64)
    k_rot = np.asarray(k_rot, np.float64)
    v = np.asarray(v, np.float64)
    sinks = np.asarray(sinks, np.float64)
    L, Hq, D = q_rot.shape
    Hkv = k_rot.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    out = np.zeros((L, Hq, D), np.float64)
    lse = np.zeros((Hq, L), np.float64)
    weights = np.zeros((Hq, L, L), np.float64) if return_weights else None
    share = np.zeros((Hq, L), np.float64) if return_weights else None
    for r0 in range(0, L, _ROW_BLOCK):
        r1 = min(L, r0 + _ROW_BLOCK)
        k0 = max(0, r0 - window + 1) if window > 0 else 0
        rows = np.arange(r0, r1)
        keys = np.arange(k0, r1)
        vis = _visible_mask(rows, keys, window)
        for h in range(Hq):
            g = h // G
            s = scale * (q_rot[r0:r1, h, :] @ k_rot[k0:r1, g, :].T)
            s = np.where(vis, s, -np.inf)
            m = np.maximum(sinks[h], s.max(axis=1))
            e = np.exp(s - m[:, None])
            e_sink = np.exp(sinks[h] - m)
            z = e_sink + e.sum(axis=1)
            out[r0:r1, h, :] = (e @ v[k0:r1, g, :]) / z[:, None]
            lse[h, r0:r1] = m + np.log(z)
            if return_weights:
                weights[h, r0:r1, k0:r1] = e / z[:, None]
                share[h, r0:r1] = e_sink / z
    if return_weights:
        return out, lse, (weights, share)
    return out, lse


def _rotate(x, positions, rope_tables):
    if rope_tables is None:
        return np.asarray(x, np.float64)
    inv_freq, conc = rope_tables
    return rope(x, positions, inv_freq, conc)


def attn_fwd_bshd(q, k, v, sinks, scale, window, rope_tables=None, positions=None):
    """BSHD prefill.  q ``[B, S, Hq, D]``, k / v ``[B, S, Hkv, D]``.

    ``rope_tables`` = ``(inv_freq, concentration)`` rotates q and k first
    (None: q and k are already rotated).  ``positions [B, S]`` default to
    0..S-1.  Returns ``out [B, S, Hq, D]`` and ``lse [B, Hq, S]``."""
    B, S = q.shape[:2]
    if positions is None:
        positions = default_positions_bshd(B, S)
    out = np.zeros(q.shape, np.float64)
    lse = np.zeros((B, q.shape[2], S), np.float64)
    for b in range(B):
        qr = _rotate(q[b], positions[b], rope_tables)
        kr = _rotate(k[b], positions[b], rope_tables)
        out[b], lse[b] = sink_attention_sequence(qr, kr, v[b], sinks, scale, window)
    return out, lse


def attn_fwd_thd(q, k, v, sinks, cu_seqlens, scale, window, rope_tables=None, positions=None):
    """Packed THD prefill.  q ``[T, Hq, D]``, k / v ``[T, Hkv, D]``,
    ``cu_seqlens [nseq + 1]``.  Positions default to restarting at 0 per
    sequence.  Returns ``out [T, Hq, D]`` and ``lse [Hq, T]``."""
    cu = np.asarray(cu_seqlens, np.int64)
    if positions is None:
        positions = default_positions_thd(cu)
    out = np.zeros(q.shape, np.float64)
    lse = np.zeros((q.shape[1], q.shape[0]), np.float64)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        qr = _rotate(q[a:b], positions[a:b], rope_tables)
        kr = _rotate(k[a:b], positions[a:b], rope_tables)
        out[a:b], lse[:, a:b] = sink_attention_sequence(qr, kr, v[a:b], sinks, scale, window)
    return out, lse


def attn_decode(q, k_cache, v_cache, cache_seqlens, sinks, scale, window, rope_tables=None):
    """Single-token decode.  q ``[B, Hq, D]`` (raw; rotated at position
    ``len_b - 1`` when ``rope_tables`` is given), caches ``[B, Lmax, Hkv, D]``
    holding post-RoPE keys and raw values, ``cache_seqlens[b] >= 1`` counts
    the new token.  The query sees cache rows ``[len_b - window, len_b)``
    (all ``[0, len_b)`` when window == 0).  Returns ``out [B, Hq, D]`` and
    ``lse [B, Hq]``."""
    q = np.asarray(q, np.float64)
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    sinks = np.asarray(sinks, np.float64)
    out = np.zeros((B, Hq, D), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    for b in range(B):
        n = int(cache_seqlens[b])
        lo = max(0, n - window) if window > 0 else 0
        qb = _rotate(q[b][None], np.array([n - 1]), rope_tables)[0]
        kb = np.asarray(k_cache[b, lo:n], np.float64)
        vb = np.asarray(v_cache[b, lo:n], np.float64)
        for h in range(Hq):
            g = h // G
            s = scale * (kb[:, g, :] @ qb[h])
            m = max(sinks[h], s.max())
            e = np.exp(s - m)
            z = np.exp(sinks[h] - m) + e.sum()
            out[b, h] = (e @ vb[:, g, :]) / z
            lse[b, h] = m + np.log(z)
    return out, lse


def attn_rows_bshd(q, k, v, sinks, scale, window, rows, rope_tables=None, positions=None):
    """Selected output rows of :func:`attn_fwd_bshd`, one by one.

    ``rows`` is a list of ``(b, h, i)``; returns ``out [n, D]`` and
    ``lse [n]``.  Used to check full-size launches on a sample."""
    B, S = q.shape[:2]
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    if positions is None:
        positions = default_positions_bshd(B, S)
    res_o = np.zeros((len(rows), q.shape[3]), np.float64)
    res_l = np.zeros(len(rows), np.float64)
    for n, (b, h, i) in enumerate(rows):
        g = h // G
        lo = max(0, i - window + 1) if window > 0 else 0
        qi = _rotate(q[b, i:i + 1, h:h + 1], positions[b, i:i + 1], rope_tables)[0, 0]
        kj = _rotate(k[b, lo:i + 1, g:g + 1], positions[b, lo:i + 1], rope_tables)[:, 0]
        vj = np.asarray(v[b, lo:i + 1, g], np.float64)
        s = scale * (kj @ qi)
        m = max(float(sinks[h]), s.max())
        e = np.exp(s - m)
        z = np.exp(float(sinks[h]) - m) + e.sum()
        res_o[n] = (e @ vj) / z
        res_l[n] = m + np.log(z)
    return res_o, res_l


def attn_rows_thd(q, k, v, sinks, cu_seqlens, scale, window, rows, rope_tables=None, positions=None):
    """Selected rows ``(t, h)`` of :func:`attn_fwd_thd`, one by one."""
    cu = np.asarray(cu_seqlens, np.int64)
    if positions is None:
        positions = default_positions_thd(cu)
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    res_o = np.zeros((len(rows), q.shape[2]), np.float64)
    res_l = np.zeros(len(rows), np.float64)
    for n, (t, h) in enumerate(rows):
        s_idx = int(np.searchsorted(cu, t, side="right") - 1)
        start = int(cu[s_idx])
        g = h // G
        lo = max(start, t - window + 1) if window > 0 else start
        qi = _rotate(q[t:t + 1, h:h + 1], positions[t:t + 1], rope_tables)[0, 0]
        kj = _rotate(k[lo:t + 1, g:g + 1], positions[lo:t + 1], rope_tables)[:, 0]
        vj = np.asarray(v[lo:t + 1, g], np.float64)
        s = scale * (kj @ qi)
        m = max(float(sinks[h]), s.max())
        e = np.exp(s - m)
        z = np.exp(float(sinks[h]) - m) + e.sum()
        res_o[n] = (e @ vj) / z
        res_l[n] = m + np.log(z)
    return res_o, res_l
