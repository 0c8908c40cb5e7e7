"""GPU parity of the paged KV cache: gptoss_attn_decode_paged against the
oracle (every output element) on scrambled block tables with garbage in the
unused pool rows, bit-identity with the contiguous decode where both cut the
keys into the same tiles, and gptoss_kv_append_paged (the rotated key within
one bf16 spacing of the exact value, the value copied, nothing else touched;
a block index outside the pool writes nothing and sets the status word)."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.paged import attn_decode_paged, kv_append_paged
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)


def _paged_case(lens, block_size, Hq=16, Hkv=2, seed=5, extra_blocks=5):
    rng = np.random.default_rng(seed)
    B = len(lens)
    max_blocks = -(-max(lens) // block_size)
    num_blocks = B * max_blocks + extra_blocks
    table = rng.permutation(num_blocks)[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    k_pool = bf16_round(rng.standard_normal((num_blocks, block_size, Hkv, 64)))
    v_pool = bf16_round(rng.standard_normal((num_blocks, block_size, Hkv, 64)))
    q = bf16_round(rng.standard_normal((B, Hq, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return q, k_pool, v_pool, table, sinks


@pytest.mark.parametrize("block_size", [64, 256])
@pytest.mark.parametrize("window", [0, 128, 100])
def test_paged_decode_matches_oracle(cuda_device, block_size, window):
    lens = [1, 77, 300, 1000, 256]
    q, kp, vp, table, sinks = _paged_case(lens, block_size)
    out, lse = ops.gptoss_attn_decode_paged(dev(q), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks),
                                            window=window, rope=ROPE, return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_decode_paged(q, kp, vp, table, block_size, lens, sinks, 0.125, window, TABLES)
    assert_parity(host(out), ref, f"paged out bs={block_size} w={window}")
    assert_lse_parity(host(lse), ref_lse, f"paged lse bs={block_size} w={window}")


def test_paged_equals_contiguous_bitwise(cuda_device):
    # full context: both paths start every split on a 64-key boundary, so they
    # see the same tiles in the same order and must agree bit for bit
    lens = [1000, 64, 513]
    bs = 128
    q, kp, vp, table, sinks = _paged_case(lens, bs, seed=9)
    L = table.shape[1] * bs
    kc = np.zeros((len(lens), L, 2, 64))
    vc = np.zeros((len(lens), L, 2, 64))
    for b, n in enumerate(lens):
        for p in range(n):
            kc[b, p] = kp[table[b, p // bs], p % bs]
            vc[b, p] = vp[table[b, p // bs], p % bs]
    got = ops.gptoss_attn_decode_paged(dev(q), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks), rope=ROPE)
    ref = ops.gptoss_attn_decode(dev(q), dev(kc), dev(vc), i32(lens), f32(sinks), rope=ROPE)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


def test_append_writes_only_the_new_rows(cuda_device):
    rng = np.random.default_rng(17)
    B, Hkv, bs, num_blocks = 4, 8, 64, 20
    table = rng.permutation(num_blocks)[:B * 4].reshape(B, 4).astype(np.int32)
    lens = [1, 64, 65, 256]  # new tokens at positions 0, 63, 64, 255
    k_new = bf16_round(rng.standard_normal((B, Hkv, 64)))
    v_new = bf16_round(rng.standard_normal((B, Hkv, 64)))
    k0 = bf16_round(rng.standard_normal((num_blocks, bs, Hkv, 64)))
    v0 = bf16_round(rng.standard_normal((num_blocks, bs, Hkv, 64)))
    kd, vd = dev(k0), dev(v0)
    ops.gptoss_kv_append_paged(dev(k_new), dev(v_new), i32(lens), i32(table), kd, vd, ROPE)
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    ref_k, ref_v = kv_append_paged(k_new, v_new, lens, table, bs, k0, v0, TABLES)
    got_k, got_v = host(kd), host(vd)
    written = np.zeros((num_blocks, bs), bool)
    for b, n in enumerate(lens):
        written[table[b, (n - 1) // bs], (n - 1) % bs] = True
    # untouched rows are bit-identical; written values: v exact, rotated k
    # within one bf16 spacing of the float64 value
    np.testing.assert_array_equal(got_k[~written], k0[~written])
    np.testing.assert_array_equal(got_v, ref_v)
    spacing = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref_k[written]), 1e-30))) - 7)
    assert np.all(np.abs(got_k[written] - ref_k[written]) <= spacing + 1e-30)


def test_append_then_decode(cuda_device):
    rng = np.random.default_rng(23)
    lens = [129, 2000, 1]
    bs = 64
    q, kp, vp, table, sinks = _paged_case(lens, bs, seed=29)
    k_new = bf16_round(rng.standard_normal((3, 2, 64)))
    v_new = bf16_round(rng.standard_normal((3, 2, 64)))
    kd, vd = dev(kp), dev(vp)
    ops.gptoss_kv_append_paged(dev(k_new), dev(v_new), i32(lens), i32(table), kd, vd, ROPE)
    out = ops.gptoss_attn_decode_paged(dev(q), kd, vd, i32(table), i32(lens), f32(sinks), rope=ROPE)
    torch.cuda.synchronize()
    # the oracle appends the exact rotation; the cache stores it in bf16, so the
    # reference decodes over the pools the device actually holds
    ref_k, ref_v = kv_append_paged(k_new, v_new, lens, table, bs, kp, vp, TABLES)
    np.testing.assert_allclose(host(kd), ref_k, rtol=2 ** -8, atol=1e-30)
    ref, _ = attn_decode_paged(q, host(kd), host(vd), table, bs, lens, sinks, 0.125, 0, TABLES)
    assert_parity(host(out), ref, "append then decode")


def test_append_out_of_range_block_writes_nothing(cuda_device):
    rng = np.random.default_rng(31)
    bs, num_blocks = 64, 4
    table = np.array([[0, 1], [2, 99]], np.int32)  # sequence 1's second block is outside the pool
    lens = [3, 70]
    k0 = bf16_round(rng.standard_normal((num_blocks, bs, 1, 64)))
    kd, vd = dev(k0), dev(k0)
    ops.read_device_status()  # clear
    ops.gptoss_kv_append_paged(dev(rng.standard_normal((2, 1, 64))), dev(rng.standard_normal((2, 1, 64))),
                               i32(lens), i32(table), kd, vd, ROPE)
    torch.cuda.synchronize()
    assert ops.read_device_status() == 1  # GPTOSS_ERR_INVALID_ARG, then cleared
    got = host(kd)
    changed = np.any(got != k0, axis=(2, 3))
    assert changed.sum() == 1 and changed[0, 2]  # only sequence 0's row (position 2) was written


@pytest.mark.parametrize("paged", [True, False])
def test_rows_past_the_end_may_hold_nan(cuda_device, paged):
    # unused cache rows (a partly filled block, slots past len) are never read
    # into the result: NaN there must not reach the output
    lens = [70, 1, 200]
    bs = 128
    q, kp, vp, table, sinks = _paged_case(lens, bs, seed=41)
    kp_nan, vp_nan = np.full_like(kp, np.nan), np.full_like(vp, np.nan)
    for b, n in enumerate(lens):
        for p in range(n):
            kp_nan[table[b, p // bs], p % bs] = kp[table[b, p // bs], p % bs]
            vp_nan[table[b, p // bs], p % bs] = vp[table[b, p // bs], p % bs]
    ref, _ = attn_decode_paged(q, kp_nan, vp_nan, table, bs, lens, sinks, 0.125, 0, TABLES)
    if paged:
        out = ops.gptoss_attn_decode_paged(dev(q), dev(kp_nan), dev(vp_nan), i32(table), i32(lens), f32(sinks),
                                           rope=ROPE)
    else:
        L = table.shape[1] * bs
        kc, vc = np.full((3, L, 2, 64), np.nan), np.full((3, L, 2, 64), np.nan)
        for b, n in enumerate(lens):
            for p in range(n):
                kc[b, p] = kp[table[b, p // bs], p % bs]
                vc[b, p] = vp[table[b, p // bs], p % bs]
        out = ops.gptoss_attn_decode(dev(q), dev(kc), dev(vc), i32(lens), f32(sinks), rope=ROPE)
    torch.cuda.synchronize()
    got = host(out)
    assert np.all(np.isfinite(got))
    assert_parity(got, ref, f"nan-padded cache paged={paged}")


# (q_len, query heads, kv heads): the tokens of a sequence share a CTA --
# G = 8: two tokens fill one 16-row fragment (q_len 2), up to four fill two
# (q_len 3), q_len 5 takes two CTAs of 4 + 1 tokens; G = 16: one token per
# fragment, two per CTA (q_len 3: 2 + 1)
@pytest.mark.parametrize("window", [0, 128])
@pytest.mark.parametrize("q_len,Hq,Hkv", [(1, 16, 2), (2, 16, 2), (3, 16, 2), (5, 16, 2), (3, 32, 2)])
def test_multi_token_decode_matches_oracle(cuda_device, window, q_len, Hq, Hkv):
    # q_len new tokens per sequence (already in the cache), each attending
    # causally; the shortest sequence holds only its new tokens
    lens = [q_len, 77, 300, 1000, 256]
    bs = 64
    q1, kp, vp, table, sinks = _paged_case(lens, bs, Hq=Hq, Hkv=Hkv, seed=43)
    rng = np.random.default_rng(47)
    q = bf16_round(rng.standard_normal((len(lens), q_len, Hq, 64)))
    out, lse = ops.gptoss_attn_decode_paged(dev(q), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks),
                                            window=window, rope=ROPE, return_lse=True)
    torch.cuda.synchronize()
    assert out.shape == (len(lens), q_len, Hq, 64) and lse.shape == (len(lens), q_len, Hq)
    ref, ref_lse = attn_decode_paged(q, kp, vp, table, bs, lens, sinks, 0.125, window, TABLES)
    assert_parity(host(out), ref, f"multi-token out q_len={q_len} G={Hq // Hkv} w={window}")
    assert_lse_parity(host(lse), ref_lse, f"multi-token lse q_len={q_len} G={Hq // Hkv} w={window}")


def test_multi_token_many_splits(cuda_device):
    # long sequences, few of them: several splits per sequence, so the merge
    # combines partials of the union range for every token
    lens = [5000, 4100, 9000]
    q_len, bs = 4, 256
    q1, kp, vp, table, sinks = _paged_case(lens, bs, seed=67)
    rng = np.random.default_rng(71)
    q = bf16_round(rng.standard_normal((len(lens), q_len, 16, 64)))
    out = ops.gptoss_attn_decode_paged(dev(q), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks), rope=ROPE)
    torch.cuda.synchronize()
    ref, _ = attn_decode_paged(q, kp, vp, table, bs, lens, sinks, 0.125, 0, TABLES)
    assert_parity(host(out), ref, "multi-token, several splits")


def test_multi_token_append_then_decode(cuda_device):
    rng = np.random.default_rng(53)
    q_len, bs = 4, 64
    lens = [4, 131, 2000]  # new tokens straddle a block edge in sequence 1 (positions 127..130)
    q1, kp, vp, table, sinks = _paged_case(lens, bs, seed=59)
    B = len(lens)
    k_new = bf16_round(rng.standard_normal((B, q_len, 2, 64)))
    v_new = bf16_round(rng.standard_normal((B, q_len, 2, 64)))
    q = bf16_round(rng.standard_normal((B, q_len, 16, 64)))
    kd, vd = dev(kp), dev(vp)
    ops.read_device_status()
    ops.gptoss_kv_append_paged(dev(k_new), dev(v_new), i32(lens), i32(table), kd, vd, ROPE)
    out = ops.gptoss_attn_decode_paged(dev(q), kd, vd, i32(table), i32(lens), f32(sinks), window=128, rope=ROPE)
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    ref_k, ref_v = kv_append_paged(k_new, v_new, lens, table, bs, kp, vp, TABLES)
    written = np.zeros(kp.shape[:2], bool)
    for b, n in enumerate(lens):
        for p in range(n - q_len, n):
            written[table[b, p // bs], p % bs] = True
    got_k = host(kd)
    np.testing.assert_array_equal(got_k[~written], kp[~written])
    np.testing.assert_array_equal(host(vd), ref_v)
    spacing = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref_k[written]), 1e-30))) - 7)
    assert np.all(np.abs(got_k[written] - ref_k[written]) <= spacing + 1e-30)
    ref, _ = attn_decode_paged(q, got_k, host(vd), table, bs, lens, sinks, 0.125, 128, TABLES)
    assert_parity(host(out), ref, "multi-token append then decode")


def test_multi_token_of_one_equals_single_token(cuda_device):
    lens = [1000, 64, 513]
    q, kp, vp, table, sinks = _paged_case(lens, 128, seed=61)
    a = ops.gptoss_attn_decode_paged(dev(q), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks), rope=ROPE)
    m = ops.gptoss_attn_decode_paged(dev(q[:, None]), dev(kp), dev(vp), i32(table), i32(lens), f32(sinks), rope=ROPE)
    torch.cuda.synchronize()
    assert torch.equal(m[:, 0], a)


def test_partial_rotary_append_then_decode(cuda_device):
    # rotary_dim 32: the appended key and the query rotate their first 32
    # features; features 32..63 are copied as given
    rng = np.random.default_rng(31)
    lens = [300, 65]
    bs = 64
    q, kp, vp, table, sinks = _paged_case(lens, bs, seed=37)
    k_new = bf16_round(rng.standard_normal((2, 2, 64)))
    v_new = bf16_round(rng.standard_normal((2, 2, 64)))
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=32)
    tabs = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0, partial_rotary_factor=0.5)
    kd, vd = dev(kp), dev(vp)
    ops.gptoss_kv_append_paged(dev(k_new), dev(v_new), i32(lens), i32(table), kd, vd, cfg)
    out = ops.gptoss_attn_decode_paged(dev(q), kd, vd, i32(table), i32(lens), f32(sinks), rope=cfg)
    torch.cuda.synchronize()
    ref_k, ref_v = kv_append_paged(k_new, v_new, lens, table, bs, kp, vp, tabs)
    np.testing.assert_allclose(host(kd), ref_k, rtol=2 ** -8, atol=1e-30)
    np.testing.assert_array_equal(host(vd), ref_v)
    ref, _ = attn_decode_paged(q, host(kd), host(vd), table, bs, lens, sinks, 0.125, 0, tabs)
    assert_parity(host(out), ref, "partial rotary append then decode")
