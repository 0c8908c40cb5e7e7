"""gptoss_attn_decode_noalloc: decode for callers that cannot allocate.

A serving loop that plans its device memory once, or a runtime that only
hands out memory from its own pools, cannot pass a freshly allocated
workspace; this entry point keeps the split-KV partials in the library's own
fixed device array instead.  The test calls it through the C ABI twice in a
row and checks each result against the workspace-taking entry point, with
the tolerance of the other parity tests.  It runs last (file name) so that a
run stopping at the first failure has already run everything else, and it
passes both alone in a fresh process and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import _abi, ops
from attention_yarn_rope_b200.workloads import DECODE_B64, GPTOSS_ROPE, make_decode_host
from tests.gpu_util import assert_parity, dev, f32, host, i32

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


@pytest.mark.parametrize("window", [0, 128])
def test_noalloc_matches_workspace_entry_twice(cuda_device, window):
    lib = _abi.load()
    lens = [2500, 1, 700, 2049]
    x = make_decode_host(DECODE_B64, B=4, L=2500, seqlens=lens, seed=201)
    q, kc, vc = dev(x.q), dev(x.k_cache), dev(x.v_cache)
    sl, sk = i32(x.seqlens), f32(x.sinks)
    rope = ops.RopeConfig.from_dict(GPTOSS_ROPE)
    ref, ref_lse = ops.gptoss_attn_decode(q, kc, vc, sl, sk, window=window, rope=rope, return_lse=True)
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((4, 64), float("nan"), dtype=torch.float32, device=cuda_device)
        st = _noalloc(lib, q, kc, vc, sl, sk, window, rope, out, lse)
        assert st == _abi.GPTOSS_OK, _abi.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        assert_parity(host(out), host(ref), f"noalloc call {call} out")
        assert_parity(host(lse), host(ref_lse), f"noalloc call {call} lse")


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
