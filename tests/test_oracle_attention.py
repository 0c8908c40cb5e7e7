"""Pins for the oracle's sink attention (CPU only).

Definition: ``GptOssAttention`` on the NeMo AutoModel ``gpt_oss.layers`` page
(``sinks``, ``sliding_window``, ``softmax_scale = head_dim ** -0.5``) and the
Transformers v4.55.0 release notes, "Architecture" (the sink adds to the
softmax denominator only; alternate full / 128-token sliding layers).

Pins, each independent of the oracle's own code:
* sink = -inf reproduces ``torch.nn.functional.scaled_dot_product_attention``
  (float64, CPU) with the GQA heads expanded, causal or with an explicit
  sliding-window mask built here;
* a sink of +60 drives the output to ~0 within a closed-form bound;
* attention weights plus the sink share sum to 1;
* a window at least as long as the sequence equals full attention (exactly);
* the first query row, which sees one key, equals v_0 (1 - share) in closed
  form;
* the brute-force formulation (scalar loops, complex RoPE, softmax over the
  logits with the sink appended as a column) agrees on tiny shapes, BSHD and
  packed THD, windows 1, 3 and longer than the sequence;
* THD equals separate per-sequence calls; decode equals the last prefill row;
  row-by-row sampling equals the full computation;
* over 1100 rows (three of the oracle's 512-row blocks, windows 0 / 1 / 128 /
  700) the output and log-sum-exp equal a whole-sequence restatement with
  ``torch.softmax`` over the logits plus a sink column and
  ``torch.logsumexp``, and with a -inf sink equal SDPA.
"""

import math

import numpy as np
import pytest
import torch

from oracle.attention import (
    attn_decode,
    attn_fwd_bshd,
    attn_fwd_thd,
    attn_rows_bshd,
    attn_rows_thd,
    sink_attention_sequence,
)
from oracle.brute import attention_concat_column
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, window):
    """Library reference: q [L,Hq,D], k/v [L,Hkv,D] -> [L,Hq,D] (float64)."""
    L, Hq, _ = q.shape
    G = Hq // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, dim=0)
    if window == 0:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    else:
        i = torch.arange(L)[:, None]
        j = torch.arange(L)[None, :]
        allowed = (j <= i) & (i - j < window)
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("window", [0, 1, 5, 16])
@pytest.mark.parametrize("hq,hkv", [(4, 1), (8, 2), (6, 6)])
def test_minus_inf_sink_is_standard_attention(window, hq, hkv):
    L, D = 37, 64
    q, k, v = _rand((L, hq, D), 1), _rand((L, hkv, D), 2), _rand((L, hkv, D), 3)
    sinks = np.full(hq, -np.inf)
    out, _ = sink_attention_sequence(q, k, v, sinks, 0.125, window)
    np.testing.assert_allclose(out, _sdpa(q, k, v, 0.125, window), rtol=1e-10, atol=1e-12)


def test_large_sink_drives_output_to_zero():
    L, D = 20, 64
    q, k, v = _rand((L, 2, D), 4), _rand((L, 1, D), 5), _rand((L, 1, D), 6)
    out, _ = sink_attention_sequence(q, k, v, np.full(2, 60.0), 0.125, 0)
    s_max = 0.125 * np.abs(q).sum(-1).max() * np.abs(k).max()
    bound = math.exp(-60.0 + s_max) * L * np.abs(v).max()
    assert bound < 1e-3
    assert np.abs(out).max() <= bound


@pytest.mark.parametrize("window", [0, 3])
def test_weights_plus_sink_share_sum_to_one(window):
    L, D = 25, 64
    q, k, v = _rand((L, 4, D), 7), _rand((L, 2, D), 8), _rand((L, 2, D), 9)
    sinks = _rand(4, 10)
    out, lse, (w, share) = sink_attention_sequence(q, k, v, sinks, 0.125, window, return_weights=True)
    np.testing.assert_allclose(w.sum(-1) + share, 1.0, rtol=0, atol=1e-12)
    # the sink share is exp(sink - lse); the output is the weighted sum of values
    np.testing.assert_allclose(share, np.exp(sinks[:, None] - lse), rtol=1e-12)
    G = 2
    recon = np.einsum("hij,jhd->ihd", w, np.repeat(v, G, axis=1))
    np.testing.assert_allclose(recon, out, rtol=1e-12, atol=1e-13)
    # masked entries have zero weight
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    hidden = (j > i) | ((window > 0) & (i - j >= window))
    assert np.all(w[:, hidden] == 0.0)


def test_window_at_least_sequence_equals_full():
    L, D = 40, 64
    q, k, v = _rand((L, 8, D), 11), _rand((L, 1, D), 12), _rand((L, 1, D), 13)
    sinks = _rand(8, 14)
    full, lse_f = sink_attention_sequence(q, k, v, sinks, 0.125, 0)
    for w in (L, L + 1, 10 * L):
        win, lse_w = sink_attention_sequence(q, k, v, sinks, 0.125, w)
        np.testing.assert_array_equal(win, full)
        np.testing.assert_array_equal(lse_w, lse_f)


def test_first_row_single_key_closed_form():
    D = 64
    q, k, v = _rand((3, 2, D), 15), _rand((3, 1, D), 16), _rand((3, 1, D), 17)
    sinks = np.array([0.3, -1.7])
    out, _ = sink_attention_sequence(q, k, v, sinks, 0.125, 0)
    for h in range(2):
        s00 = 0.125 * float(q[0, h] @ k[0, 0])
        share = math.exp(sinks[h]) / (math.exp(sinks[h]) + math.exp(s00))
        np.testing.assert_allclose(out[0, h], v[0, 0] * (1.0 - share), rtol=1e-13)


def _nested(a):
    return a.tolist()


@pytest.mark.parametrize("window", [0, 1, 3, 21])
def test_brute_force_agreement_bshd_with_yarn(window):
    L, Hq, Hkv, D = 16, 4, 2, 64
    q, k, v = _rand((1, L, Hq, D), 20), _rand((1, L, Hkv, D), 21), _rand((1, L, Hkv, D), 22)
    sinks = _rand(Hq, 23)
    out, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=TABLES)
    inv, conc = TABLES
    bo, _ = attention_concat_column(_nested(q[0]), _nested(k[0]), _nested(v[0]), list(sinks), 0.125, window,
                                    [(0, L)], list(range(L)), list(inv), conc)
    np.testing.assert_allclose(out[0], np.array(bo), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("window", [0, 2, 9])
def test_brute_force_agreement_thd(window):
    lens = [5, 1, 7]
    cu = np.array([0, 5, 6, 13])
    T, Hq, Hkv, D = 13, 4, 2, 64
    q, k, v = _rand((T, Hq, D), 30), _rand((T, Hkv, D), 31), _rand((T, Hkv, D), 32)
    sinks = _rand(Hq, 33)
    sinks[1] = -np.inf
    out, _ = attn_fwd_thd(q, k, v, sinks, cu, 0.125, window, rope_tables=TABLES)
    pos = [p for n in lens for p in range(n)]
    inv, conc = TABLES
    bo, _ = attention_concat_column(_nested(q), _nested(k), _nested(v), list(sinks), 0.125, window,
                                    [(0, 5), (5, 6), (6, 13)], pos, list(inv), conc)
    np.testing.assert_allclose(out, np.array(bo), rtol=1e-12, atol=1e-12)


def test_thd_equals_separate_sequences():
    cu = np.array([0, 9, 20, 21, 30])
    T, Hq, Hkv, D = 30, 8, 2, 64
    q, k, v = _rand((T, Hq, D), 40), _rand((T, Hkv, D), 41), _rand((T, Hkv, D), 42)
    sinks = _rand(Hq, 43)
    out, lse = attn_fwd_thd(q, k, v, sinks, cu, 0.125, 4, rope_tables=TABLES)
    for s in range(4):
        a, b = cu[s], cu[s + 1]
        o1, l1 = attn_fwd_bshd(q[None, a:b], k[None, a:b], v[None, a:b], sinks, 0.125, 4, rope_tables=TABLES)
        np.testing.assert_array_equal(out[a:b], o1[0])
        np.testing.assert_array_equal(lse[:, a:b], l1[0])


@pytest.mark.parametrize("window", [0, 6])
def test_decode_equals_last_prefill_row(window):
    B, L, Hq, Hkv, D = 3, 23, 8, 2, 64
    q, k, v = _rand((B, L, Hq, D), 50), _rand((B, L, Hkv, D), 51), _rand((B, L, Hkv, D), 52)
    sinks = _rand(Hq, 53)
    lens = np.array([23, 1, 11])
    inv, conc = TABLES
    k_cache = np.zeros((B, L, Hkv, D))
    v_cache = np.zeros((B, L, Hkv, D))
    for b in range(B):
        k_cache[b] = rope(k[b], np.arange(L), inv, conc)
        v_cache[b] = v[b]
    q_new = np.stack([q[b, lens[b] - 1] for b in range(B)])
    out, lse = attn_decode(q_new, k_cache, v_cache, lens, sinks, 0.125, window, rope_tables=TABLES)
    for b in range(B):
        n = lens[b]
        ref, ref_lse = attn_fwd_bshd(q[b:b + 1, :n], k[b:b + 1, :n], v[b:b + 1, :n], sinks, 0.125, window,
                                     rope_tables=TABLES)
        np.testing.assert_allclose(out[b], ref[0, n - 1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], ref_lse[0, :, n - 1], rtol=1e-12)


@pytest.mark.parametrize("window", [0, 7])
def test_row_sampling_matches_full(window):
    B, S, Hq, Hkv, D = 2, 40, 4, 2, 64
    q, k, v = _rand((B, S, Hq, D), 60), _rand((B, S, Hkv, D), 61), _rand((B, S, Hkv, D), 62)
    sinks = _rand(Hq, 63)
    out, lse = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=TABLES)
    rows = [(0, 0, 0), (1, 3, 39), (0, 2, 17), (1, 1, 6)]
    ro, rl = attn_rows_bshd(q, k, v, sinks, 0.125, window, rows, rope_tables=TABLES)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(ro[n], out[b, i, h], rtol=1e-12, atol=1e-13)
        assert rl[n] == pytest.approx(lse[b, h, i], rel=1e-12)
    cu = np.array([0, 15, 40])
    qt, kt, vt = q[0], k[0], v[0]
    out_t, lse_t = attn_fwd_thd(qt, kt, vt, sinks, cu, 0.125, window, rope_tables=TABLES)
    rows_t = [(0, 0), (14, 3), (15, 1), (39, 2)]
    ro, rl = attn_rows_thd(qt, kt, vt, sinks, cu, 0.125, window, rows_t, rope_tables=TABLES)
    for n, (t, h) in enumerate(rows_t):
        np.testing.assert_allclose(ro[n], out_t[t, h], rtol=1e-12, atol=1e-13)
        assert rl[n] == pytest.approx(lse_t[h, t], rel=1e-12)


def _torch_sink_attention(q, k, v, sinks, scale, window):
    """The definition restated with library routines over the whole sequence
    at once: a full [L, L] logit matrix, the visibility mask built from
    index grids, the sink as one more softmax column (``torch.softmax``) and
    the log-sum-exp from ``torch.logsumexp``.  float64, CPU."""
    L, Hq, _ = q.shape
    G = Hq // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, dim=0)
    logits = scale * qt @ kt.transpose(1, 2)
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    allowed = j <= i
    if window > 0:
        allowed = allowed & (i - j < window)
    logits = logits.masked_fill(~allowed, float("-inf"))
    col = torch.from_numpy(np.asarray(sinks, np.float64)).view(Hq, 1, 1).expand(Hq, L, 1)
    full = torch.cat([logits, col], dim=-1)
    w = torch.softmax(full, dim=-1)[..., :L]
    return (w @ vt).permute(1, 0, 2).numpy(), torch.logsumexp(full, dim=-1).numpy()


@pytest.mark.parametrize("window", [0, 1, 128, 700])
def test_several_row_blocks_against_library_softmax(window):
    # 1100 rows span three of the oracle's 512-row blocks; the band of the
    # later blocks starts at r0 - window + 1, which this pins row by row
    L, Hq, Hkv, D = 1100, 4, 2, 64
    q, k, v = _rand((L, Hq, D), 70), _rand((L, Hkv, D), 71), _rand((L, Hkv, D), 72)
    sinks = _rand(Hq, 73)
    out, lse = sink_attention_sequence(q, k, v, sinks, 0.125, window)
    ref_o, ref_l = _torch_sink_attention(q, k, v, sinks, 0.125, window)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-13, atol=0)
    # and the row-by-row path on the rows around the block edges
    pos = np.arange(L)
    rows = [(0, h, i) for h in (0, 3) for i in (0, 511, 512, 513, 639, 640, 1023, 1024, 1099)]
    ro, rl = attn_rows_bshd(q[None], k[None], v[None], sinks, 0.125, window, rows, positions=pos[None])
    for n, (_, h, i) in enumerate(rows):
        np.testing.assert_allclose(ro[n], out[i, h], rtol=0, atol=1e-12)
        assert rl[n] == pytest.approx(lse[h, i], rel=1e-13)


@pytest.mark.parametrize("window", [0, 128])
def test_several_row_blocks_minus_inf_sink_is_sdpa(window):
    L, Hq, Hkv, D = 1100, 2, 1, 64
    q, k, v = _rand((L, Hq, D), 74), _rand((L, Hkv, D), 75), _rand((L, Hkv, D), 76)
    out, _ = sink_attention_sequence(q, k, v, np.full(Hq, -np.inf), 0.125, window)
    np.testing.assert_allclose(out, _sdpa(q, k, v, 0.125, window), rtol=0, atol=1e-12)
