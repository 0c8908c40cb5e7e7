"""Out-of-bounds writes: every entry point's outputs and workspace handed out
as the interior of canary-padded buffers (tests/canary_util.py), with ragged
shapes that end mid-tile; after the call every sentinel must be intact and
every output finite.  Values are checked by the parity tests; this file
checks only where the kernels write."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from tests.canary_util import Canvas, HeadCanvas
from tests.gpu_util import dev, f32, i32

pytestmark = pytest.mark.gpu

ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)
BF = torch.bfloat16
F32 = torch.float32
U8 = torch.uint8


def _bf(rng, shape):
    return dev(bf16_round(rng.standard_normal(shape)))


def _ok(*canvases):
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    for c in canvases:
        assert c.intact(), type(c).__name__
        t = c.t.float() if c.t.dtype != U8 else None
        if t is not None:
            assert bool(torch.isfinite(t).all())


@pytest.mark.parametrize("window", [0, 128])
def test_prefill_bshd(cuda_device, window):
    rng = np.random.default_rng(201)
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v = _bf(rng, (B, S, Hq, 64)), _bf(rng, (B, S, Hkv, 64)), _bf(rng, (B, S, Hkv, 64))
    sinks = f32(rng.standard_normal(Hq))
    out = Canvas((B, S, Hq, 64), BF, cuda_device)
    lse = Canvas((B, Hq, S), F32, cuda_device)
    ws = Canvas((ops.gptoss_attn_fwd_workspace_size(B * S, Hkv),), U8, cuda_device)
    ops.gptoss_attn_fwd(q, k, v, sinks, window=window, rope=ROPE, out=out.t, lse=lse.t, workspace=ws.t)
    _ok(out, lse)
    assert ws.intact()
    # a strided output whose neighbouring heads are sentinels
    outh = HeadCanvas(B, S, Hq, 64, cuda_device)
    ops.gptoss_attn_fwd(q, k, v, sinks, window=window, rope=ROPE, out=outh.t)
    _ok(outh)


def test_prefill_thd(cuda_device):
    rng = np.random.default_rng(203)
    cu = [0, 1, 78, 378, 449]  # lengths 1, 77, 300, 71
    T, Hq, Hkv = cu[-1], 16, 2
    q, k, v = _bf(rng, (T, Hq, 64)), _bf(rng, (T, Hkv, 64)), _bf(rng, (T, Hkv, 64))
    sinks = f32(rng.standard_normal(Hq))
    out = Canvas((T, Hq, 64), BF, cuda_device)
    lse = Canvas((Hq, T), F32, cuda_device)
    ops.gptoss_attn_fwd(q, k, v, sinks, window=128, rope=ROPE, cu_seqlens=i32(cu), max_seqlen=300, out=out.t,
                        lse=lse.t)
    _ok(out, lse)


def test_rope(cuda_device):
    rng = np.random.default_rng(205)
    B, S, Hq, Hkv = 2, 77, 16, 2
    q, k = _bf(rng, (B, S, Hq, 64)), _bf(rng, (B, S, Hkv, 64))
    qo = Canvas((B, S, Hq, 64), BF, cuda_device)
    ko = Canvas((B, S, Hkv, 64), BF, cuda_device)
    ops.gptoss_rope_qk(q, k, ROPE, q_out=qo.t, k_out=ko.t)
    _ok(qo, ko)


@pytest.mark.parametrize("window", [0, 128])
def test_decode(cuda_device, window):
    rng = np.random.default_rng(207)
    lens = [1, 513, 1000]
    B, L, Hq, Hkv = len(lens), 1000, 16, 2
    q = _bf(rng, (B, Hq, 64))
    kc, vc = _bf(rng, (B, L, Hkv, 64)), _bf(rng, (B, L, Hkv, 64))
    out = Canvas((B, Hq, 64), BF, cuda_device)
    lse = Canvas((B, Hq), F32, cuda_device)
    ws = Canvas((ops.gptoss_attn_decode_workspace_size(B, L, Hq, Hkv),), U8, cuda_device)
    ops.gptoss_attn_decode(q, kc, vc, i32(lens), f32(rng.standard_normal(Hq)), window=window, rope=ROPE, out=out.t,
                           lse=lse.t, workspace=ws.t)
    _ok(out, lse)
    assert ws.intact()


def test_paged_multi_token_decode(cuda_device):
    rng = np.random.default_rng(209)
    lens, q_len, bs = [3, 200, 513], 3, 64
    B, Hq, Hkv = len(lens), 16, 2
    max_blocks = -(-max(lens) // bs)
    num_blocks = B * max_blocks + 3
    table = rng.permutation(num_blocks)[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    kp, vp = _bf(rng, (num_blocks, bs, Hkv, 64)), _bf(rng, (num_blocks, bs, Hkv, 64))
    q = _bf(rng, (B, q_len, Hq, 64))
    out = Canvas((B, q_len, Hq, 64), BF, cuda_device)
    lse = Canvas((B, q_len, Hq), F32, cuda_device)
    ws = Canvas((ops.gptoss_attn_decode_workspace_size(B * q_len, max_blocks * bs, Hq, Hkv),), U8, cuda_device)
    ops.gptoss_attn_decode_paged(q, kp, vp, i32(table), i32(lens), f32(rng.standard_normal(Hq)), window=0, rope=ROPE,
                                 out=out.t, lse=lse.t, workspace=ws.t)
    _ok(out, lse)
    assert ws.intact()


# (S, window): the sliding path (mma.sync dQ, direct dK / dV), and full
# context long enough to split the dK / dV sweeps (tcgen05 dQ, fp32 accumulators)
@pytest.mark.parametrize("S,window", [(300, 128), (1100, 0)])
def test_backward(cuda_device, S, window):
    rng = np.random.default_rng(211)
    B, Hq, Hkv = 1, 16, 2
    q, k, v = _bf(rng, (B, S, Hq, 64)), _bf(rng, (B, S, Hkv, 64)), _bf(rng, (B, S, Hkv, 64))
    sinks = f32(rng.standard_normal(Hq))
    out, lse = ops.gptoss_attn_fwd(q, k, v, sinks, window=window, rope=ROPE, return_lse=True)
    dout = _bf(rng, (B, S, Hq, 64))
    dq = Canvas((B, S, Hq, 64), BF, cuda_device)
    dk = Canvas((B, S, Hkv, 64), BF, cuda_device)
    dv = Canvas((B, S, Hkv, 64), BF, cuda_device)
    ds = Canvas((Hq,), F32, cuda_device)
    ws = Canvas((ops.gptoss_attn_bwd_workspace_size(B * S, Hq, Hkv),), U8, cuda_device)
    ops.gptoss_attn_bwd(q, k, v, sinks, out, dout, lse, window=window, rope=ROPE, dq=dq.t, dk=dk.t, dv=dv.t,
                        dsinks=ds.t, workspace=ws.t)
    _ok(dq, dk, dv, ds)
    assert ws.intact()
