"""Paged KV cache: decode over it and appending to it (test infrastructure only).

The pages describe autoregressive generation with a key/value cache
(Transformers v4.55.0 release notes: the ``model.generate`` examples, the
cache entries of the change list) but give no cache layout.  This module
follows the layout the CUDA path implements (a block table over a pool of
fixed-size blocks, the common paged layout) and reduces both operations to
the plain definitions in :mod:`oracle.attention` and :mod:`oracle.rope`:

* token ``p`` of sequence ``b`` lives in block ``block_table[b][p // bs]`` at
  row ``p % bs`` of the pools ``[num_blocks, bs, Hkv, D]``;
* decode over the pool is :func:`oracle.attention.attn_decode` over the rows
  gathered into a contiguous cache;
* appending the new token of sequence ``b`` (position ``len_b - 1``, the new
  token counted in ``len_b``) writes its key rotated at that position (the
  cache holds post-RoPE keys) and its value as given.

Several new tokens per sequence (``q_len``: draft tokens checked in one pass;
the pages' generation examples take one token a step, so this is the plain
extension of causal attention to them): token ``i`` sits at position
``len_b - q_len + i``, is appended like a single token at that position, and
its query sees exactly the keys a causal prefill row at that position sees --
the cache rows ``[0, len_b - q_len + i]`` (windowed as usual).  Decoding it is
:func:`oracle.attention.attn_decode` with the length cut to
``len_b - (q_len - 1 - i)``.

Plain NumPy, float64 unless stated; imports nothing from the CUDA package.
"""

from __future__ import annotations

import numpy as np

from .attention import attn_decode
from .rope import rope


def gather_paged(pool, block_table_row, block_size: int, n: int) -> np.ndarray:
    """Rows ``[0, n)`` of one sequence, in token order, from a paged pool."""
    out = np.empty((n,) + pool.shape[2:], pool.dtype)
    for p in range(n):
        out[p] = pool[int(block_table_row[p // block_size]), p % block_size]
    return out


def attn_decode_paged(q, k_pool, v_pool, block_table, block_size, cache_seqlens, sinks, scale, window,
                      rope_tables=None):
    """Decode over a paged cache.  ``q [B, Hq, D]`` (one new token per
    sequence) gives ``out [B, Hq, D]``, ``lse [B, Hq]``; ``q [B, q_len, Hq, D]``
    (q_len new tokens, all already in the cache) gives ``out [B, q_len, Hq,
    D]``, ``lse [B, q_len, Hq]``, token i seeing ``len_b - (q_len - 1 - i)``
    cache rows.  Every ``len_b`` must be at least ``q_len``."""
    q = np.asarray(q, np.float64)
    multi = q.ndim == 4
    q4 = q if multi else q[:, None]
    B, q_len = q4.shape[:2]
    lens = [int(x) for x in cache_seqlens]
    if min(lens) < q_len:
        raise ValueError("every sequence must hold its q_len new tokens")
    lmax = max(lens)
    Hkv, D = k_pool.shape[2], k_pool.shape[3]
    kc = np.zeros((B, lmax, Hkv, D), np.float64)
    vc = np.zeros((B, lmax, Hkv, D), np.float64)
    for b in range(B):
        kc[b, :lens[b]] = gather_paged(k_pool, block_table[b], block_size, lens[b])
        vc[b, :lens[b]] = gather_paged(v_pool, block_table[b], block_size, lens[b])
    out = np.zeros(q4.shape, np.float64)
    lse = np.zeros(q4.shape[:3], np.float64)
    for i in range(q_len):
        lens_i = [n - (q_len - 1 - i) for n in lens]
        out[:, i], lse[:, i] = attn_decode(q4[:, i], kc, vc, lens_i, sinks, scale, window, rope_tables=rope_tables)
    return (out, lse) if multi else (out[:, 0], lse[:, 0])


def kv_append_paged(k_new, v_new, cache_seqlens, block_table, block_size, k_pool, v_pool, rope_tables):
    """Copies of the pools with each sequence's new tokens written.  ``k_new``
    / ``v_new`` are ``[B, Hkv, D]`` (one token) or ``[B, q_len, Hkv, D]``;
    token i's key is rotated at position ``len_b - q_len + i``, its value
    stored as given.  Returns float64 pools; the CUDA path stores bf16."""
    k_new = np.asarray(k_new, np.float64)
    v_new = np.asarray(v_new, np.float64)
    if k_new.ndim == 3:
        k_new, v_new = k_new[:, None], v_new[:, None]
    kp = np.array(k_pool, np.float64)
    vp = np.array(v_pool, np.float64)
    B, q_len = k_new.shape[:2]
    for b in range(B):
        for i in range(q_len):
            pos = int(cache_seqlens[b]) - q_len + i
            blk = int(block_table[b][pos // block_size])
            row = pos % block_size
            kp[blk, row] = rope(k_new[b, i][None], np.array([pos]), *rope_tables)[0]
            vp[blk, row] = v_new[b, i]
    return kp, vp
