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
    """Single-token decode over a paged cache: ``out [B, Hq, D]``, ``lse [B, Hq]``."""
    B = q.shape[0]
    lens = [int(x) for x in cache_seqlens]
    lmax = max(lens)
    Hkv, D = k_pool.shape[2], k_pool.shape[3]
    kc = np.zeros((B, lmax, Hkv, D), np.float64)
    vc = np.zeros((B, lmax, Hkv, D), np.float64)
    for b in range(B):
        kc[b, :lens[b]] = gather_paged(k_pool, block_table[b], block_size, lens[b])
        vc[b, :lens[b]] = gather_paged(v_pool, block_table[b], block_size, lens[b])
    return attn_decode(q, kc, vc, lens, sinks, scale, window, rope_tables=rope_tables)


def kv_append_paged(k_new, v_new, cache_seqlens, block_table, block_size, k_pool, v_pool, rope_tables):
    """Copies of the pools with each sequence's new token written: the key
    ``k_new[b]`` (``[Hkv, D]``) rotated at position ``len_b - 1``, the value
    ``v_new[b]`` as given.  Returns float64 pools; the CUDA path stores bf16."""
    kp = np.array(k_pool, np.float64)
    vp = np.array(v_pool, np.float64)
    for b in range(k_new.shape[0]):
        pos = int(cache_seqlens[b]) - 1
        blk = int(block_table[b][pos // block_size])
        row = pos % block_size
        k_rot = rope(np.asarray(k_new[b], np.float64)[None], np.array([pos]), *rope_tables)[0]
        kp[blk, row] = k_rot
        vp[blk, row] = np.asarray(v_new[b], np.float64)
    return kp, vp
