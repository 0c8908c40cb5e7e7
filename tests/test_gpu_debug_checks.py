"""The range-checking build (libgptoss_attn_debug.so, GPTOSS_DEBUG_CHECKS).

Its kernels check the indices they compute from device-side data --
cu_seqlens (nondecreasing, within the T tokens, no sequence longer than the
stated maximum), cache_seqlens (1 <= len <= Lmax) and the logical
coordinates of every output row -- and a failed check records
GPTOSS_ERR_INVALID_ARG in the device status word while the access is
skipped; nothing traps.  Here the build runs small parity cases against the
float64 oracle with a clean status word, then malformed cu_seqlens and
cache_seqlens: the status word reports them, the well-formed sequences are
still correct and rows of skipped sequences are left untouched.  Only the
debug build is given malformed inputs.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import _abi, ops
from attention_yarn_rope_b200.workloads import DECODE_B64, GPTOSS_ROPE, bf16_round, make_decode_host
from oracle.attention import attn_decode, attn_fwd_bshd, attn_fwd_thd
from oracle.rope import default_positions_thd, rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, bf16_ulp, dev, f32, host, i32

pytestmark = pytest.mark.gpu

TABS = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)


def _rand(shape, seed):
    return bf16_round(np.random.default_rng(seed).standard_normal(shape))


@pytest.fixture
def debug_lib(cuda_device):
    saved = _abi._lib
    _abi._lib = _abi.load_debug()
    ops.read_device_status(reset=True)
    try:
        yield
    finally:
        _abi._lib = saved


def test_debug_build_parity(debug_lib):
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v = _rand((B, S, Hq, 64), 1), _rand((B, S, Hkv, 64), 2), _rand((B, S, Hkv, 64), 3)
    sinks = np.random.default_rng(4).standard_normal(Hq).astype(np.float32)
    out, lse = ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=128, rope=ROPE, return_lse=True)
    lens = [1, 129, 170]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    qt, kt, vt = q[0], k[0], v[0]
    out_t = ops.gptoss_attn_fwd(dev(qt), dev(kt), dev(vt), f32(sinks), window=0, cu_seqlens=i32(cu),
                                max_seqlen=max(lens), rope=ROPE)
    x = make_decode_host(DECODE_B64, B=3, L=700, seqlens=[700, 1, 333], seed=5)
    out_d = ops.gptoss_attn_decode(dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(x.seqlens), f32(x.sinks),
                                   window=0, rope=ROPE)
    qo, ko = ops.gptoss_rope_qk(dev(qt), dev(kt), ROPE, cu_seqlens=i32(cu))
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    ref, ref_l = attn_fwd_bshd(q, k, v, sinks, 0.125, 128, rope_tables=TABS)
    assert_parity(host(out), ref, "debug build prefill out")
    assert_lse_parity(host(lse), ref_l, "debug build prefill lse")
    ref_t, _ = attn_fwd_thd(qt, kt, vt, sinks, cu, 0.125, 0, rope_tables=TABS)
    assert_parity(host(out_t), ref_t, "debug build thd out")
    ref_d, _ = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, 0.125, 0, rope_tables=TABS)
    assert_parity(host(out_d), ref_d, "debug build decode out")
    pos = default_positions_thd(cu)
    ref_q = rope(qt, pos, *TABS)
    assert np.all(np.abs(host(qo) - ref_q) <= bf16_ulp(ref_q) + 1e-6)


def test_debug_build_flags_bad_cu_seqlens(debug_lib):
    # T = 300 tokens; the second entry runs past T and the third goes backwards:
    # only sequence 0 ([0, 100)) is well formed
    T, Hq, Hkv = 300, 8, 1
    cu = np.array([0, 100, 400, 300], np.int32)
    q, k, v = _rand((T, Hq, 64), 6), _rand((T, Hkv, 64), 7), _rand((T, Hkv, 64), 8)
    sinks = np.random.default_rng(9).standard_normal(Hq).astype(np.float32)
    out = torch.full((T, Hq, 64), 7.0, dtype=torch.bfloat16, device="cuda:0")
    ops.gptoss_attn_fwd(dev(q), dev(k), dev(v), f32(sinks), window=0, cu_seqlens=i32(cu), max_seqlen=300,
                        rope=ROPE, out=out)
    torch.cuda.synchronize()
    assert ops.read_device_status() == _abi.GPTOSS_ERR_INVALID_ARG
    ref, _ = attn_fwd_thd(q[:100], k[:100], v[:100], sinks, np.array([0, 100]), 0.125, 0, rope_tables=TABS)
    o = host(out)
    assert_parity(o[:100], ref, "well-formed sequence next to malformed ones")
    assert np.all(o[100:] == 7.0)  # the skipped sequences' rows are untouched


def test_debug_build_flags_cache_longer_than_lmax(debug_lib):
    x = make_decode_host(DECODE_B64, B=2, L=500, seqlens=[300, 500], seed=10)
    lens = np.array([300, 600], np.int32)  # sequence 1 claims more rows than the cache holds
    out = ops.gptoss_attn_decode(dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(lens), f32(x.sinks), window=0,
                                 rope=ROPE)
    torch.cuda.synchronize()
    assert ops.read_device_status() == _abi.GPTOSS_ERR_INVALID_ARG
    ref, _ = attn_decode(x.q[:1], x.k_cache[:1], x.v_cache[:1], [300], x.sinks, 0.125, 0, rope_tables=TABS)
    assert_parity(host(out[:1]), ref, "well-formed sequence next to a malformed one")
