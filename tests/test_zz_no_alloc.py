"""gptoss_attn_decode_noalloc: decode for callers that cannot allocate.

A serving loop that plans its device memory once, or a runtime that only
hands out memory from its own pools, cannot pass a freshly allocated
workspace; this entry point keeps the split-KV partials in the library's own
fixed device array instead.  The test calls it through the C ABI twice in a
row and checks each result against the float64 oracle on the same seeded
inputs and against the workspace-taking entry point, with the tolerance of
the other parity tests.  Between the two checked calls it makes a no-alloc
call of another shape (more sequences, longer caches, more key splits), so a
call that read partials left in the shared array by an earlier call would
change the second result.  It runs last (file name) so that a
run stopping at the first failure has already run everything else, and it
passes both alone in a fresh process and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import _abi, ops
from attention_yarn_rope_b200.workloads import DECODE_B64, GPTOSS_ROPE, make_decode_host
from oracle.attention import attn_decode
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, kc, vc, lens, sinks, window, rope, out, lse):
    B, Hq, D = q.shape
    _, L, Hkv, _ = kc.shape
    r = rope.to_c()
    return lib.gptoss_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(lens.data_ptr()), ctypes.c_void_p(sinks.data_ptr()), B, L, Hq, Hkv, D, window, 0.125,
        ctypes.byref(r), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _tables():
    r = GPTOSS_ROPE
    return yarn_inv_freq_and_concentration(64, r["base"], r["factor"], r["initial_context"], r["ntk_alpha"],
                                           r["ntk_beta"])


@pytest.mark.parametrize("window", [0, 128])
def test_noalloc_matches_oracle_and_workspace_entry_twice(cuda_device, window):
    lib = _abi.load()
    lens = [2500, 1, 700, 2049]
    x = make_decode_host(DECODE_B64, B=4, L=2500, seqlens=lens, seed=201)
    q, kc, vc = dev(x.q), dev(x.k_cache), dev(x.v_cache)
    sl, sk = i32(x.seqlens), f32(x.sinks)
    rope = ops.RopeConfig.from_dict(GPTOSS_ROPE)
    ora_o, ora_l = attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, 0.125, window, rope_tables=_tables())
    ref, ref_lse = ops.gptoss_attn_decode(q, kc, vc, sl, sk, window=window, rope=rope, return_lse=True)
    torch.cuda.synchronize()
    # another shape in between: 8 sequences of up to 20000 keys, more splits
    lens2 = [20000, 9000, 1, 17000, 20000, 333, 12000, 5000]
    y = make_decode_host(DECODE_B64, B=8, L=20000, seqlens=lens2, seed=202)
    q2, kc2, vc2 = dev(y.q), dev(y.k_cache), dev(y.v_cache)
    sl2, sk2 = i32(y.seqlens), f32(y.sinks)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((4, 64), float("nan"), dtype=torch.float32, device=cuda_device)
        st = _noalloc(lib, q, kc, vc, sl, sk, window, rope, out, lse)
        assert st == _abi.GPTOSS_OK, _abi.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        assert_parity(host(out), ora_o, f"noalloc call {call} out vs oracle")
        assert_lse_parity(host(lse), ora_l, f"noalloc call {call} lse vs oracle")
        assert_parity(host(out), host(ref), f"noalloc call {call} out vs workspace entry")
        assert_lse_parity(host(lse), host(ref_lse), f"noalloc call {call} lse vs workspace entry")
        if call == 0:
            out2 = torch.full_like(q2, float("nan"))
            lse2 = torch.full((8, 64), float("nan"), dtype=torch.float32, device=cuda_device)
            st = _noalloc(lib, q2, kc2, vc2, sl2, sk2, window, rope, out2, lse2)
            assert st == _abi.GPTOSS_OK, _abi.STATUS_NAMES.get(st, st)
            torch.cuda.synchronize()
            o2, l2 = attn_decode(y.q, y.k_cache, y.v_cache, y.seqlens, y.sinks, 0.125, window, rope_tables=_tables())
            assert_parity(host(out2), o2, "noalloc, second shape, out vs oracle")
            assert_lse_parity(host(lse2), l2, "noalloc, second shape, lse vs oracle")


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    lib = _abi.load()
    # 64 sequences x 131072 slots need 33 MiB of partials, above the 16 MiB array
    assert ops.gptoss_attn_decode_workspace_size(64, 131072, 64, 8) > (16 << 20)
    fake = torch.empty(16, dtype=torch.uint8, device=cuda_device)
    p = ctypes.c_void_p(fake.data_ptr())
    r = ops.RopeConfig.from_dict(GPTOSS_ROPE).to_c()
    st = lib.gptoss_attn_decode_noalloc(p, p, p, p, p, 64, 131072, 64, 8, 64, 0, 0.125, ctypes.byref(r), p, None,
                                        None)
    assert st == _abi.GPTOSS_ERR_UNSUPPORTED
