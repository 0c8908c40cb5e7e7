"""Pins of the paged-cache oracle (oracle/paged.py) on the CPU: a paged pool
with any block permutation decodes exactly like the contiguous cache it was
scattered from; the appended key sits in the right block row and equals an
independent (complex-multiply) rotation; append-then-decode equals decode over
the contiguous cache that holds the rotated new key; several new tokens per
sequence, appended and decoded, reproduce the last rows of a causal prefill
over the whole sequence (a different code path: the prefill's row mask)."""

import numpy as np
import pytest

from oracle.attention import attn_decode, attn_fwd_bshd
from oracle.brute import rope_complex
from oracle.paged import attn_decode_paged, gather_paged, kv_append_paged
from oracle.yarn import yarn_inv_freq_and_concentration

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _scatter(cache, lens, block_size, rng, extra_blocks=3):
    """Pools holding `cache` [B, L, Hkv, D] under a random block permutation."""
    B, L = cache.shape[:2]
    nb_seq = -(-L // block_size)
    nblocks = B * nb_seq + extra_blocks
    perm = rng.permutation(nblocks)
    table = perm[:B * nb_seq].reshape(B, nb_seq)
    pool = rng.standard_normal((nblocks, block_size) + cache.shape[2:])  # garbage everywhere else
    for b in range(B):
        for p in range(lens[b]):
            pool[table[b, p // block_size], p % block_size] = cache[b, p]
    return pool, table


@pytest.mark.parametrize("block_size,window", [(64, 0), (128, 0), (64, 50), (16, 7)])
def test_paged_decode_equals_contiguous(block_size, window):
    rng = np.random.default_rng(7)
    B, L, Hq, Hkv, D = 3, 300, 4, 2, 64
    lens = [1, 170, 300]
    kc, vc = rng.standard_normal((B, L, Hkv, D)), rng.standard_normal((B, L, Hkv, D))
    q, sinks = rng.standard_normal((B, Hq, D)), rng.standard_normal(Hq)
    kp, table = _scatter(kc, lens, block_size, rng)
    vp = np.array(kp)  # same table for the values (rows outside the sequences stay garbage)
    for b in range(B):
        for p in range(lens[b]):
            vp[table[b, p // block_size], p % block_size] = vc[b, p]
    got_o, got_l = attn_decode_paged(q, kp, vp, table, block_size, lens, sinks, 0.125, window, TABLES)
    ref_o, ref_l = attn_decode(q, kc, vc, lens, sinks, 0.125, window, TABLES)
    np.testing.assert_array_equal(got_o, ref_o)
    np.testing.assert_array_equal(got_l, ref_l)


def test_gather_follows_the_table():
    pool = np.arange(5 * 4).reshape(5, 4, 1, 1).astype(np.float64)  # block k, row r holds 4k + r
    rows = gather_paged(pool, [3, 0, 4], 4, 10)[:, 0, 0]
    np.testing.assert_array_equal(rows, [12, 13, 14, 15, 0, 1, 2, 3, 16, 17])


def test_append_writes_rotated_key_and_raw_value():
    rng = np.random.default_rng(11)
    B, Hkv, D, bs = 3, 2, 64, 16
    nblocks = 12
    table = np.array([[5, 2, 9], [0, 7, 1], [11, 3, 4]])
    lens = [1, 17, 48]  # new tokens at positions 0, 16, 47
    k_new, v_new = rng.standard_normal((B, Hkv, D)), rng.standard_normal((B, Hkv, D))
    kp0 = np.zeros((nblocks, bs, Hkv, D))
    kp, vp = kv_append_paged(k_new, v_new, lens, table, bs, kp0, kp0, TABLES)
    written = {(5, 0), (7, 0), (4, 15)}  # (block, row) of positions 0, 16, 47
    for blk in range(nblocks):
        for row in range(bs):
            assert (np.any(kp[blk, row] != 0)) == ((blk, row) in written)
    inv, c = TABLES
    for b, (blk, row) in enumerate([(5, 0), (7, 0), (4, 15)]):
        pos = lens[b] - 1
        for g in range(Hkv):
            np.testing.assert_allclose(kp[blk, row, g], rope_complex(k_new[b, g], pos, inv, c), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(vp[blk, row], v_new[b])


def test_append_then_decode_equals_contiguous():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, D, bs, L = 2, 4, 1, 64, 32, 96
    lens = [40, 96]
    kc, vc = rng.standard_normal((B, L, Hkv, D)), rng.standard_normal((B, L, Hkv, D))
    q, sinks = rng.standard_normal((B, Hq, D)), rng.standard_normal(Hq)
    k_new, v_new = rng.standard_normal((B, Hkv, D)), rng.standard_normal((B, Hkv, D))
    table = np.array([[2, 0, 5], [1, 4, 3]])
    kp = np.zeros((6, bs, Hkv, D))
    vp = np.zeros((6, bs, Hkv, D))
    for b in range(B):
        for p in range(lens[b] - 1):
            kp[table[b, p // bs], p % bs] = kc[b, p]
            vp[table[b, p // bs], p % bs] = vc[b, p]
    kp, vp = kv_append_paged(k_new, v_new, lens, table, bs, kp, vp, TABLES)
    got, _ = attn_decode_paged(q, kp, vp, table, bs, lens, sinks, 0.125, 0, TABLES)
    inv, c = TABLES
    for b in range(B):
        for g in range(Hkv):
            kc[b, lens[b] - 1, g] = rope_complex(k_new[b, g], lens[b] - 1, inv, c)
        vc[b, lens[b] - 1] = v_new[b]
    ref, _ = attn_decode(q, kc, vc, lens, sinks, 0.125, 0, TABLES)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [0, 5, 128])
def test_multi_token_append_and_decode_equal_prefill_rows(window):
    # a sequence of L tokens whose first L - q_len keys are already cached
    # (rotated by the brute-force complex rotation); append the last q_len raw
    # keys, decode the last q_len raw queries: the result is the causal prefill
    # of all L tokens at rows L - q_len .. L - 1
    rng = np.random.default_rng(19)
    B, L, q_len, Hq, Hkv, D, bs = 2, 70, 4, 4, 2, 64, 16
    q = rng.standard_normal((B, L, Hq, D))
    k = rng.standard_normal((B, L, Hkv, D))
    v = rng.standard_normal((B, L, Hkv, D))
    sinks = rng.standard_normal(Hq)
    ref_o, ref_l = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=TABLES)
    nb_seq = -(-L // bs)
    table = rng.permutation(B * nb_seq + 2)[:B * nb_seq].reshape(B, nb_seq)
    kp = rng.standard_normal((B * nb_seq + 2, bs, Hkv, D))
    vp = rng.standard_normal((B * nb_seq + 2, bs, Hkv, D))
    inv, c = TABLES
    for b in range(B):
        for p in range(L - q_len):
            for g in range(Hkv):
                kp[table[b, p // bs], p % bs, g] = rope_complex(k[b, p, g], p, inv, c)
            vp[table[b, p // bs], p % bs] = v[b, p]
    lens = [L] * B
    kp, vp = kv_append_paged(k[:, L - q_len:], v[:, L - q_len:], lens, table, bs, kp, vp, TABLES)
    got_o, got_l = attn_decode_paged(q[:, L - q_len:], kp, vp, table, bs, lens, sinks, 0.125, window, TABLES)
    assert got_o.shape == (B, q_len, Hq, D) and got_l.shape == (B, q_len, Hq)
    np.testing.assert_allclose(got_o, ref_o[:, L - q_len:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_l, np.transpose(ref_l, (0, 2, 1))[:, L - q_len:], rtol=0, atol=1e-12)


def test_multi_token_with_one_token_is_single_token_decode():
    rng = np.random.default_rng(21)
    B, Hq, Hkv, D, bs = 2, 4, 2, 64, 32
    lens = [33, 64]
    table = np.array([[1, 0], [3, 2]])
    kp, vp = rng.standard_normal((4, bs, Hkv, D)), rng.standard_normal((4, bs, Hkv, D))
    q, sinks = rng.standard_normal((B, Hq, D)), rng.standard_normal(Hq)
    a = attn_decode_paged(q, kp, vp, table, bs, lens, sinks, 0.125, 0, TABLES)
    m = attn_decode_paged(q[:, None], kp, vp, table, bs, lens, sinks, 0.125, 0, TABLES)
    np.testing.assert_array_equal(m[0][:, 0], a[0])
    np.testing.assert_array_equal(m[1][:, 0], a[1])


def test_multi_token_needs_its_tokens_in_the_cache():
    z = np.zeros((2, 32, 1, 64))
    with pytest.raises(ValueError):
        attn_decode_paged(np.zeros((1, 3, 1, 64)), z, z, np.array([[0]]), 32, [2], np.zeros(1), 0.125, 0)
