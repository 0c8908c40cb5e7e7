"""GPU parity of gptoss_attn_decode (split-KV decode) against the oracle.

Small caches compared on every output element: ragged lengths (1, a split
boundary, the full cache), full and 128 windows, GPT-OSS head grouping,
sinks -inf / large, queries rotated at the true position.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import DECODE_B64, GPTOSS_ROPE, make_decode_host
from oracle.attention import attn_decode
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


@pytest.mark.parametrize("window", [0, 128, 1])
def test_decode_ragged(cuda_device, window):
    L = 3000
    lens = [3000, 1, 517, 256, 2049, 129]
    x = make_decode_host(DECODE_B64, B=len(lens), L=L, seqlens=lens, seed=101)
    out, lse = ops.gptoss_attn_decode(dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(x.seqlens), f32(x.sinks),
                                      window=window, rope=ops.RopeConfig.from_dict(GPTOSS_ROPE), return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, 0.125, window, rope_tables=TABLES)
    assert_parity(host(out), ref, f"decode out w={window}")
    assert_lse_parity(host(lse), ref_lse, f"decode lse w={window}")


@pytest.mark.parametrize("sink", [-np.inf, 25.0])
def test_decode_extreme_sinks_no_rope(cuda_device, sink):
    lens = [700, 64, 65]
    x = make_decode_host(DECODE_B64, B=3, L=700, seqlens=lens, seed=102)
    sinks = np.full(64, sink, np.float32)
    sinks[3] = -1.0
    out = ops.gptoss_attn_decode(dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(x.seqlens), f32(sinks), window=0)
    torch.cuda.synchronize()
    ref, _ = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, sinks, 0.125, 0, rope_tables=None)
    assert_parity(host(out), ref, f"decode sink={sink}")


def test_decode_reuses_workspace_and_is_deterministic(cuda_device):
    lens = [1500, 900]
    x = make_decode_host(DECODE_B64, B=2, L=1500, seqlens=lens, seed=103)
    args = (dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(x.seqlens), f32(x.sinks))
    ws = torch.empty(ops.gptoss_attn_decode_workspace_size(2, 1500, 64, 8), dtype=torch.uint8, device=cuda_device)
    ws.fill_(0xFF)  # garbage (NaN patterns) must not leak into the result
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE)
    o1 = ops.gptoss_attn_decode(*args, window=0, rope=cfg, workspace=ws)
    o2 = ops.gptoss_attn_decode(*args, window=0, rope=cfg, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    ref, _ = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, 0.125, 0, rope_tables=TABLES)
    assert_parity(host(o1), ref, "decode ws reuse")


@pytest.mark.parametrize("rotary_dim", [16, 32])
@pytest.mark.parametrize("window", [0, 128])
def test_decode_partial_rotary(cuda_device, rotary_dim, window):
    # partial_rotary_factor = rotary_dim / 64: the query rotates its first
    # rotary_dim features only (the cache holds keys rotated the same way)
    lens = [900, 1, 300]
    x = make_decode_host(DECODE_B64, B=3, L=900, seqlens=lens, seed=104 + rotary_dim)
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=rotary_dim)
    out, lse = ops.gptoss_attn_decode(dev(x.q), dev(x.k_cache), dev(x.v_cache), i32(x.seqlens), f32(x.sinks),
                                      window=window, rope=cfg, return_lse=True)
    torch.cuda.synchronize()
    tabs = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0,
                                           partial_rotary_factor=rotary_dim / 64)
    ref, ref_lse = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, 0.125, window, rope_tables=tabs)
    assert_parity(host(out), ref, f"decode partial rotary {rotary_dim} out")
    assert_lse_parity(host(lse), ref_lse, f"decode partial rotary {rotary_dim} lse")
