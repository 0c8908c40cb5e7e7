"""GPU parity of gptoss_attn_fwd (prefill) against the float64 oracle.

Every element of out (and lse) is compared, at sizes the oracle finishes in
seconds but that span several 128-row tiles and a ragged tail: BSHD and
packed THD, full and sliding windows (1, 128, 200, longer than the sequence),
RoPE fused or inputs pre-rotated, default and explicit positions, sinks of
-inf, +large and N(0,1), and the tiny correctness workload.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, PLAIN_ROPE, TINY, bf16_round, make_prefill
from oracle.attention import attn_fwd_bshd, attn_fwd_thd
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu


def _tables(rp):
    return yarn_inv_freq_and_concentration(64, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                           rp["ntk_beta"])


def _rand(shape, seed):
    return bf16_round(np.random.default_rng(seed).standard_normal(shape))


def test_tiny_workload(cuda_device):
    x = make_prefill(TINY)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=TINY.window,
                                   rope=ops.RopeConfig.from_dict(TINY.rope), return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_fwd_bshd(x.q, x.k, x.v, x.sinks, TINY.softmax_scale, TINY.window,
                                 rope_tables=_tables(TINY.rope))
    assert_parity(host(out), ref, "tiny out")
    assert_lse_parity(host(lse), ref_lse, "tiny lse")


# rope modes: RoPE fused into the call, or q and k rotated beforehand (no
# RoPE in the call)
ROPE_MODES = ["fused", "prerotated"]


@pytest.mark.parametrize("window", [0, 1, 128, 200, 1000])
@pytest.mark.parametrize("mode", ROPE_MODES)
def test_bshd_multi_tile_ragged(cuda_device, window, mode):
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v = _rand((B, S, Hq, 64), 1), _rand((B, S, Hkv, 64), 2), _rand((B, S, Hkv, 64), 3)
    sinks = np.random.default_rng(4).standard_normal(Hq).astype(np.float32)
    tabs = _tables(GPTOSS_ROPE)
    if mode != "prerotated":
        out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=window,
                                       rope=ops.RopeConfig.from_dict(GPTOSS_ROPE), return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=tabs)
    else:
        # pre-rotated bf16 inputs: both sides get the oracle's rotation rounded to bf16
        pos = np.broadcast_to(np.arange(S), (B, S))
        qr = np.stack([bf16_round(rope(q[b], pos[b], *tabs)) for b in range(B)])
        kr = np.stack([bf16_round(rope(k[b], pos[b], *tabs)) for b in range(B)])
        out, lse = ops.gptoss_attn_fwd(dev(qr), dev(kr), dev(v), f32(sinks), window=window, return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = attn_fwd_bshd(qr, kr, v, sinks, 0.125, window, rope_tables=None)
    assert_parity(host(out), ref, f"out w={window}")
    assert_lse_parity(host(lse), ref_lse, f"lse w={window}")


@pytest.mark.parametrize("sink", [-np.inf, 30.0])
def test_extreme_sinks(cuda_device, sink):
    B, S, Hq, Hkv = 1, 256, 8, 1
    q, k, v = _rand((B, S, Hq, 64), 11), _rand((B, S, Hkv, 64), 12), _rand((B, S, Hkv, 64), 13)
    sinks = np.full(Hq, sink, np.float32)
    sinks[1] = 0.5
    out = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), rope=ops.RopeConfig.from_dict(PLAIN_ROPE))
    torch.cuda.synchronize()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, 0, rope_tables=_tables(PLAIN_ROPE))
    assert_parity(host(out), ref, f"sink={sink}")


@pytest.mark.parametrize("window", [0, 128])
def test_thd_ragged_sequences(cuda_device, window):
    lens = [1, 129, 300, 77, 128, 256]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv = int(cu[-1]), 16, 2
    q, k, v = _rand((T, Hq, 64), 21), _rand((T, Hkv, 64), 22), _rand((T, Hkv, 64), 23)
    sinks = np.random.default_rng(24).standard_normal(Hq).astype(np.float32)
    out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=window, cu_seqlens=i32(cu),
                                   max_seqlen=max(lens), rope=ops.RopeConfig.from_dict(GPTOSS_ROPE),
                                   return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_fwd_thd(q, k, v, sinks, cu, 0.125, window, rope_tables=_tables(GPTOSS_ROPE))
    assert_parity(host(out), ref, "thd out")
    assert_lse_parity(host(lse), ref_lse, "thd lse")


def test_explicit_positions_and_strided_io(cuda_device):
    # q/k/v as views of one fused buffer; output into a strided view; positions offset by a prefix
    B, S, Hq, Hkv = 2, 200, 8, 2
    qkv = _rand((B, S, Hq + 2 * Hkv, 64), 31)
    t = dev(qkv)
    q, k, v = t[:, :, :Hq], t[:, :, Hq:Hq + Hkv], t[:, :, Hq + Hkv:]
    sinks = np.random.default_rng(32).standard_normal(Hq).astype(np.float32)
    pos = (np.arange(S)[None, :] + np.array([[1000], [130000]])).astype(np.int32)
    big = torch.zeros((B, S, Hq + 8, 64), dtype=torch.bfloat16, device=cuda_device)
    out = big[:, :, 4:4 + Hq]
    ops.gptoss_attn_fwd(q, k, v, f32(sinks), window=128, rope=ops.RopeConfig.from_dict(GPTOSS_ROPE),
                        positions=i32(pos), out=out)
    torch.cuda.synchronize()
    ref, _ = attn_fwd_bshd(qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:], sinks, 0.125, 128,
                           rope_tables=_tables(GPTOSS_ROPE), positions=pos)
    assert_parity(host(out), ref, "strided out")
    assert float(big[:, :, :4].abs().max()) == 0.0 and float(big[:, :, 4 + Hq:].abs().max()) == 0.0


def test_gpt_oss_head_layout_two_tiles(cuda_device):
    # the production head counts (64 / 8) on a short sequence, full causal
    B, S, Hq, Hkv = 1, 256, 64, 8
    q, k, v = _rand((B, S, Hq, 64), 41), _rand((B, S, Hkv, 64), 42), _rand((B, S, Hkv, 64), 43)
    sinks = np.random.default_rng(44).standard_normal(Hq).astype(np.float32)
    out = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), rope=ops.RopeConfig.from_dict(GPTOSS_ROPE))
    torch.cuda.synchronize()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, 0, rope_tables=_tables(GPTOSS_ROPE))
    assert_parity(host(out), ref, "gpt-oss heads")


@pytest.mark.parametrize("rotary_dim", [16, 32, 48])
@pytest.mark.parametrize("window", [0, 128])
def test_partial_rotary(cuda_device, rotary_dim, window):
    # partial_rotary_factor = rotary_dim / 64: q and k rotate their first
    # rotary_dim features in pairs (j, j + rotary_dim / 2); the rest pass through
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v = _rand((B, S, Hq, 64), 51), _rand((B, S, Hkv, 64), 52), _rand((B, S, Hkv, 64), 53)
    sinks = np.random.default_rng(54).standard_normal(Hq).astype(np.float32)
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=rotary_dim)
    out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=window, rope=cfg, return_lse=True)
    torch.cuda.synchronize()
    tabs = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0,
                                           partial_rotary_factor=rotary_dim / 64)
    ref, ref_lse = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=tabs)
    assert_parity(host(out), ref, f"partial rotary {rotary_dim} out w={window}")
    assert_lse_parity(host(lse), ref_lse, f"partial rotary {rotary_dim} lse w={window}")


def test_partial_rotary_thd_explicit_positions(cuda_device):
    lens = [1, 200, 77]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv = int(cu[-1]), 8, 2
    q, k, v = _rand((T, Hq, 64), 55), _rand((T, Hkv, 64), 56), _rand((T, Hkv, 64), 57)
    sinks = np.random.default_rng(58).standard_normal(Hq).astype(np.float32)
    pos = np.random.default_rng(59).integers(0, 131072, T).astype(np.int32)
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=32)
    out = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=128, cu_seqlens=i32(cu),
                              max_seqlen=max(lens), rope=cfg, positions=i32(pos))
    torch.cuda.synchronize()
    tabs = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0, partial_rotary_factor=0.5)
    ref, _ = attn_fwd_thd(q, k, v, sinks, cu, 0.125, 128, rope_tables=tabs, positions=pos)
    assert_parity(host(out), ref, "partial rotary thd out")
