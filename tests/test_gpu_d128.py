"""GPU parity at head size D = 128 (the variant with twice GPT-OSS's head
size) against the float64 oracle: gptoss_rope_qk with full and partial
rotary, and the prefill (gptoss_attn_fwd) with RoPE fused or inputs
pre-rotated, full and sliding windows, BSHD with a ragged last tile, packed
THD, explicit positions and extreme sinks; decode over a contiguous cache
(full and 128 windows, full and partial rotary) and over a paged cache after
appending 1 or 3 new tokens.  Every element of out and lse is compared
against the same bar as at D = 64."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.attention import attn_fwd_bshd, attn_fwd_thd
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu

D = 128
SCALE = D ** -0.5


def _tables(rotary_dim=D):
    rp = GPTOSS_ROPE
    return yarn_inv_freq_and_concentration(rotary_dim, rp["base"], rp["factor"], rp["initial_context"],
                                           rp["ntk_alpha"], rp["ntk_beta"])


def _rope_cfg(rotary_dim=D):
    return ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=rotary_dim)


def _rand(shape, seed):
    return bf16_round(np.random.default_rng(seed).standard_normal(shape))


@pytest.mark.parametrize("rotary_dim", [128, 64])
def test_rope_qk_d128(cuda_device, rotary_dim):
    B, S, Hq, Hkv = 2, 300, 4, 2
    q, k = _rand((B, S, Hq, D), 1), _rand((B, S, Hkv, D), 2)
    qo, ko = ops.gptoss_rope_qk(dev(q), dev(k), _rope_cfg(rotary_dim))
    torch.cuda.synchronize()
    tabs = _tables(rotary_dim)
    pos = np.arange(S)
    for b in range(B):
        for got, x in ((qo, q), (ko, k)):
            ref = rope(x[b], pos, *tabs)
            err = np.abs(host(got)[b] - ref)
            # one bf16 spacing of the result (the output is bf16)
            spacing = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
            assert np.all(err <= spacing + 1e-6), float(err.max())
    if rotary_dim < D:  # features past the rotary ones pass through unchanged
        assert np.array_equal(host(qo)[..., rotary_dim:], q[..., rotary_dim:])


@pytest.mark.parametrize("window", [0, 1, 128, 200])
@pytest.mark.parametrize("mode", ["fused", "prerotated"])
def test_prefill_d128_bshd_ragged(cuda_device, window, mode):
    B, S, Hq, Hkv = 2, 300, 6, 2
    q, k, v = _rand((B, S, Hq, D), 11), _rand((B, S, Hkv, D), 12), _rand((B, S, Hkv, D), 13)
    sinks = np.random.default_rng(14).standard_normal(Hq).astype(np.float32)
    tabs = _tables()
    if mode == "fused":
        out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=window, rope=_rope_cfg(),
                                       return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = attn_fwd_bshd(q, k, v, sinks, SCALE, window, rope_tables=tabs)
    else:
        pos = np.arange(S)
        qr = np.stack([bf16_round(rope(q[b], pos, *tabs)) for b in range(B)])
        kr = np.stack([bf16_round(rope(k[b], pos, *tabs)) for b in range(B)])
        out, lse = ops.gptoss_attn_fwd(dev(qr), dev(kr), dev(v), f32(sinks), window=window, return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = attn_fwd_bshd(qr, kr, v, sinks, SCALE, window, rope_tables=None)
    assert_parity(host(out), ref, f"D=128 out w={window} {mode}")
    assert_lse_parity(host(lse), ref_lse, f"D=128 lse w={window} {mode}")


@pytest.mark.parametrize("window", [0, 128])
def test_prefill_d128_thd(cuda_device, window):
    lens = [1, 129, 300, 77, 256]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv = int(cu[-1]), 8, 1
    q, k, v = _rand((T, Hq, D), 21), _rand((T, Hkv, D), 22), _rand((T, Hkv, D), 23)
    sinks = np.random.default_rng(24).standard_normal(Hq).astype(np.float32)
    out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=window, cu_seqlens=i32(cu),
                                   max_seqlen=max(lens), rope=_rope_cfg(), return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_fwd_thd(q, k, v, sinks, cu, SCALE, window, rope_tables=_tables())
    assert_parity(host(out), ref, "D=128 thd out")
    assert_lse_parity(host(lse), ref_lse, "D=128 thd lse")


def test_prefill_d128_explicit_positions_extreme_sinks(cuda_device):
    B, S, Hq, Hkv = 2, 260, 4, 1
    q, k, v = _rand((B, S, Hq, D), 31), _rand((B, S, Hkv, D), 32), _rand((B, S, Hkv, D), 33)
    sinks = np.array([-np.inf, 30.0, 0.0, -2.0], np.float32)
    pos = (np.arange(S)[None, :] + np.array([[1000], [130000]])).astype(np.int32)
    out = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=128, rope=_rope_cfg(), positions=i32(pos))
    torch.cuda.synchronize()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, SCALE, 128, rope_tables=_tables(), positions=pos)
    assert_parity(host(out), ref, "D=128 explicit positions")


def test_prefill_d128_rejects_partial_rotary(cuda_device):
    q = torch.zeros((1, 128, 2, D), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((1, 128, 1, D), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        ops.gptoss_attn_fwd(q, k, k, torch.zeros(2, device=cuda_device), rope=_rope_cfg(64))


# ---------------------------------------------------------------- decode, D = 128
def _decode_case(lens, Hq=8, Hkv=2, seed=41):
    rng = np.random.default_rng(seed)
    B, L = len(lens), max(lens)
    q = bf16_round(rng.standard_normal((B, Hq, D)))
    kc = bf16_round(rng.standard_normal((B, L, Hkv, D)))
    vc = bf16_round(rng.standard_normal((B, L, Hkv, D)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return q, kc, vc, np.array(lens, np.int32), sinks


@pytest.mark.parametrize("window", [0, 128])
@pytest.mark.parametrize("rotary_dim", [128, 64])
def test_decode_d128(cuda_device, window, rotary_dim):
    from oracle.attention import attn_decode
    q, kc, vc, lens, sinks = _decode_case([3000, 1, 517, 129, 2049])
    out, lse = ops.gptoss_attn_decode(dev(q), dev(kc), dev(vc), i32(lens), f32(sinks), window=window,
                                      rope=_rope_cfg(rotary_dim), return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_decode(q, kc, vc, lens, sinks, SCALE, window, rope_tables=_tables(rotary_dim))
    assert_parity(host(out), ref, f"D=128 decode w={window} r={rotary_dim}")
    assert_lse_parity(host(lse), ref_lse, f"D=128 decode lse w={window} r={rotary_dim}")


@pytest.mark.parametrize("q_len", [1, 3])
def test_paged_append_then_decode_d128(cuda_device, q_len):
    from oracle.paged import attn_decode_paged, kv_append_paged
    rng = np.random.default_rng(43)
    lens = [129, 2000, 5]
    bs, Hq, Hkv = 64, 16, 2
    B = len(lens)
    max_blocks = -(-max(lens) // bs)
    num_blocks = B * max_blocks + 3
    table = rng.permutation(num_blocks)[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    kp = bf16_round(rng.standard_normal((num_blocks, bs, Hkv, D)))
    vp = bf16_round(rng.standard_normal((num_blocks, bs, Hkv, D)))
    q = bf16_round(rng.standard_normal((B, q_len, Hq, D)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    k_new = bf16_round(rng.standard_normal((B, q_len, Hkv, D)))
    v_new = bf16_round(rng.standard_normal((B, q_len, Hkv, D)))
    kd, vd = dev(kp), dev(vp)
    ops.gptoss_kv_append_paged(dev(k_new), dev(v_new), i32(lens), i32(table), kd, vd, _rope_cfg())
    out, lse = ops.gptoss_attn_decode_paged(dev(q), kd, vd, i32(table), i32(lens), f32(sinks), window=128,
                                            rope=_rope_cfg(), return_lse=True)
    torch.cuda.synchronize()
    ref_k, ref_v = kv_append_paged(k_new, v_new, lens, table, bs, kp, vp, _tables())
    np.testing.assert_allclose(host(kd), ref_k, rtol=2 ** -8, atol=1e-30)
    np.testing.assert_array_equal(host(vd), ref_v)
    ref, ref_lse = attn_decode_paged(q, host(kd), host(vd), table, bs, lens, sinks, SCALE, 128, _tables())
    assert_parity(host(out), ref, f"D=128 paged q_len={q_len}")
    assert_lse_parity(host(lse), ref_lse, f"D=128 paged lse q_len={q_len}")
