"""GPU parity of gptoss_qkv_rope (q, k, v projections with RoPE in the GEMM
epilogue) against the float64 oracle (oracle/projection.py), every output
element: GPT-OSS's projection sizes (hidden 2880, 64 / 8 heads of 64) over
several 128-token tiles with a ragged tail, BSHD and packed THD, explicit
positions, no bias and no RoPE, and head size 128.

Bar: each output is the fp32-accumulated product rounded to bf16, so an
element may differ from the float64 value by half a bf16 spacing of the
result (at most |ref| 2^-8: bf16 keeps 8 significant bits) plus the fp32
accumulation and table error (1e-3 absolute here: the
outputs are O(1))."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.projection import qkv_rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import dev, host, i32

pytestmark = pytest.mark.gpu


def _tabs(D):
    rp = GPTOSS_ROPE
    return yarn_inv_freq_and_concentration(D, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                           rp["ntk_beta"])


def _weights(Hq, Hkv, D, hidden, seed):
    rng = np.random.default_rng(seed)
    N = (Hq + 2 * Hkv) * D
    # Linear-like scales: outputs of unit size
    return bf16_round(rng.standard_normal((N, hidden)) / np.sqrt(hidden)), bf16_round(rng.standard_normal(N) * 0.1)


def _check(got, ref, what):
    got = host(got)
    err = np.abs(got - ref)
    bar = np.abs(ref) * 2.0 ** -8 + 1e-3  # half a bf16 spacing: |ref| 2^-8 at most
    i = np.unravel_index(np.argmax(err - bar), err.shape)
    assert np.all(err <= bar), f"{what}: err {err[i]:.3g} at {i} (ref {ref[i]:.4g}), max abs {err.max():.3g}"


@pytest.mark.parametrize("use_rope", [True, False])
def test_gpt_oss_projection_bshd(cuda_device, use_rope):
    B, S, hidden, Hq, Hkv, D = 2, 300, 2880, 64, 8, 64
    w, b = _weights(Hq, Hkv, D, hidden, 1)
    x = bf16_round(np.random.default_rng(2).standard_normal((B, S, hidden)))
    rope = ops.RopeConfig.from_dict(GPTOSS_ROPE) if use_rope else None
    q, k, v = ops.gptoss_qkv_rope(dev(x), dev(w), dev(b), Hq, Hkv, rope=rope)
    torch.cuda.synchronize()
    pos = np.tile(np.arange(S), B)
    rq, rk, rv = qkv_rope(x.reshape(B * S, hidden), w, b, pos, Hq, Hkv, D,
                          rope_tables=_tabs(D) if use_rope else None)
    _check(q.reshape(B * S, Hq, D), rq, "q")
    _check(k.reshape(B * S, Hkv, D), rk, "k")
    _check(v.reshape(B * S, Hkv, D), rv, "v")


def test_thd_explicit_positions_no_bias(cuda_device):
    lens = [130, 1, 257, 40]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, hidden, Hq, Hkv, D = int(cu[-1]), 512, 16, 2, 64
    w, _ = _weights(Hq, Hkv, D, hidden, 3)
    x = bf16_round(np.random.default_rng(4).standard_normal((T, hidden)))
    pos = np.random.default_rng(5).integers(0, 131072, T).astype(np.int32)
    q, k, v = ops.gptoss_qkv_rope(dev(x), dev(w), None, Hq, Hkv, rope=ops.RopeConfig.from_dict(GPTOSS_ROPE),
                                  positions=i32(pos), cu_seqlens=i32(cu))
    torch.cuda.synchronize()
    rq, rk, rv = qkv_rope(x, w, None, pos, Hq, Hkv, D, rope_tables=_tabs(D))
    _check(q, rq, "q")
    _check(k, rk, "k")
    _check(v, rv, "v")


def test_head_dim_128(cuda_device):
    B, S, hidden, Hq, Hkv, D = 1, 200, 1024, 8, 2, 128
    w, b = _weights(Hq, Hkv, D, hidden, 6)
    x = bf16_round(np.random.default_rng(7).standard_normal((B, S, hidden)))
    q, k, v = ops.gptoss_qkv_rope(dev(x), dev(w), dev(b), Hq, Hkv,
                                  rope=ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=D))
    torch.cuda.synchronize()
    rq, rk, rv = qkv_rope(x.reshape(S, hidden), w, b, np.arange(S), Hq, Hkv, D, rope_tables=_tabs(D))
    _check(q.reshape(S, Hq, D), rq, "q")
    _check(k.reshape(S, Hkv, D), rk, "k")
    _check(v.reshape(S, Hkv, D), rv, "v")


def test_projection_feeds_attention(cuda_device):
    # the fused projection's q / k / v go straight into the prefill (pre-rotated, no RoPE in the call)
    from oracle.attention import attn_fwd_bshd
    from tests.gpu_util import assert_parity, f32
    B, S, hidden, Hq, Hkv, D = 1, 256, 2880, 64, 8, 64
    w, b = _weights(Hq, Hkv, D, hidden, 8)
    x = bf16_round(np.random.default_rng(9).standard_normal((B, S, hidden)))
    sinks = np.random.default_rng(10).standard_normal(Hq).astype(np.float32)
    q, k, v = ops.gptoss_qkv_rope(dev(x), dev(w), dev(b), Hq, Hkv, rope=ops.RopeConfig.from_dict(GPTOSS_ROPE))
    out = ops.gptoss_attn_fwd(q, k, v, f32(sinks), window=128)
    torch.cuda.synchronize()
    ref = attn_fwd_bshd(host(q), host(k), host(v), sinks, 0.125, 128, rope_tables=None)[0]
    assert_parity(host(out), ref, "projection -> attention")
