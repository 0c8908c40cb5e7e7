"""Pins of the key-block attention and log-sum-exp merge (oracle/cp.py) on
the CPU: any split of a sequence's keys into blocks, merged, is the prefill
oracle of the whole sequence (full context and windows, GQA heads, RoPE at
global positions); the merge does not depend on the blocks' order; a block
no row can see changes nothing; a -inf sink is standard softmax over the
blocks."""

import numpy as np
import pytest

from oracle.attention import attn_fwd_bshd
from oracle.cp import block_attention, merge_blocks
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
SCALE = 0.125


def _case(rng, S, Hq=4, Hkv=2):
    return (rng.standard_normal((1, S, Hq, 64)), rng.standard_normal((1, S, Hkv, 64)),
            rng.standard_normal((1, S, Hkv, 64)), rng.standard_normal(Hq))


def _rotated(q, k):
    pos = np.arange(q.shape[1])
    return rope(q[0], pos, *TABLES), rope(k[0], pos, *TABLES)


@pytest.mark.parametrize("window,cuts", [(0, [0, 37, 80, 150]), (0, [0, 1, 149, 150]), (20, [0, 50, 100, 150]),
                                         (1, [0, 75, 150])])
def test_query_shards_over_key_blocks_equal_the_prefill(window, cuts):
    rng = np.random.default_rng(31)
    S = cuts[-1]
    q, k, v, sinks = _case(rng, S)
    ref_o, ref_l = attn_fwd_bshd(q, k, v, sinks, SCALE, window, rope_tables=TABLES)
    qr, kr = _rotated(q, k)
    # every query shard against every key shard that is not after it, merged
    for a in range(len(cuts) - 1):
        q0, q1 = cuts[a], cuts[a + 1]
        parts = [block_attention(qr[q0:q1], kr[k0:k1], v[0, k0:k1], SCALE, window, q0, k0)
                 for k0, k1 in zip(cuts[:a + 1], cuts[1:a + 2])]
        o, lse = merge_blocks(parts, sinks)
        np.testing.assert_allclose(o, ref_o[0, q0:q1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l[0, :, q0:q1], rtol=0, atol=1e-12)


def test_merge_is_order_free_and_ignores_blind_blocks():
    rng = np.random.default_rng(37)
    q, k, v, sinks = _case(rng, 90)
    qr, kr = _rotated(q, k)
    parts = [block_attention(qr[60:90], kr[a:b], v[0, a:b], SCALE, 0, 60, a) for a, b in ((0, 30), (30, 60), (60, 90))]
    o1, l1 = merge_blocks(parts, sinks)
    o2, l2 = merge_blocks(parts[::-1], sinks)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    # a later key block is invisible to these rows: lse -inf, no effect on the merge
    blind = block_attention(qr[0:30], kr[60:90], v[0, 60:90], SCALE, 0, 0, 60)
    assert np.all(blind[1] == -np.inf) and np.all(blind[0] == 0)
    base = merge_blocks([block_attention(qr[0:30], kr[0:30], v[0, 0:30], SCALE, 0, 0, 0)], sinks)
    with_blind = merge_blocks([block_attention(qr[0:30], kr[0:30], v[0, 0:30], SCALE, 0, 0, 0), blind], sinks)
    np.testing.assert_array_equal(base[0], with_blind[0])
    np.testing.assert_array_equal(base[1], with_blind[1])


def test_minus_inf_sink_is_plain_softmax_over_the_blocks():
    rng = np.random.default_rng(41)
    q, k, v, _ = _case(rng, 64)
    sinks = np.full(4, -np.inf)
    qr, kr = _rotated(q, k)
    parts = [block_attention(qr[32:64], kr[a:b], v[0, a:b], SCALE, 0, 32, a) for a, b in ((0, 32), (32, 64))]
    o, lse = merge_blocks(parts, sinks)
    # direct softmax over all visible keys of rows 32..63
    for h in range(4):
        s = SCALE * qr[32:64, h] @ kr[:, h // 2].T
        s[np.arange(64)[None, :] > 32 + np.arange(32)[:, None]] = -np.inf  # row 32 + r sees keys 0 .. 32 + r
        w = np.exp(s - s.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(o[:, h], w @ v[0, :, h // 2], rtol=0, atol=1e-12)
