"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: every output element (and every lse) against the float64
oracle, for all of

* sliding-window prefill B=4, S=4096, 64/8 heads, window 128, YaRN RoPE;
* full-context prefill B=2, S=8192 (about a minute of oracle time on a few
  host cores);
* the packed THD stream of 32768 tokens, full context and window 128;
* decode B=64 x 32768 and B=8 x 131072, full and window 128, every sequence
  (caches drawn on the device and read back one sequence at a time).
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import (
    DECODE_B8,
    DECODE_B8_W,
    DECODE_B64,
    DECODE_B64_W,
    FULL,
    SLIDING,
    THD_FULL,
    THD_WINDOW,
    make_decode_device,
    make_prefill,
)
from oracle.attention import attn_decode, attn_fwd_bshd, attn_fwd_thd
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu


def _tables(rp):
    return yarn_inv_freq_and_concentration(64, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                           rp["ntk_beta"])


def test_sliding_prefill_full_size_every_element(cuda_device):
    cfg = SLIDING
    x = make_prefill(cfg)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=cfg.window,
                                   rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    o, l = host(out), host(lse)
    del out, lse
    ref_o, ref_l = attn_fwd_bshd(x.q, x.k, x.v, x.sinks, cfg.softmax_scale, cfg.window, rope_tables=_tables(cfg.rope))
    assert_parity(o, ref_o, cfg.name + " out (every element)")
    assert_lse_parity(l, ref_l, cfg.name + " lse (every element)")


def test_full_prefill_full_size_every_element(cuda_device):
    cfg = FULL
    x = make_prefill(cfg)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=cfg.window,
                                   rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    o, l = host(out), host(lse)
    del out, lse
    ref_o, ref_l = attn_fwd_bshd(x.q, x.k, x.v, x.sinks, cfg.softmax_scale, cfg.window, rope_tables=_tables(cfg.rope))
    assert_parity(o, ref_o, cfg.name + " out (every element)")
    assert_lse_parity(l, ref_l, cfg.name + " lse (every element)")


def _thd_call(cfg):
    x = make_prefill(cfg)
    cu = x.cu_seqlens
    lens = np.diff(cu)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=cfg.window,
                                   cu_seqlens=i32(cu), max_seqlen=int(lens.max()),
                                   rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    return x, host(out), host(lse)


def test_thd_window_full_size_every_element(cuda_device):
    cfg = THD_WINDOW
    x, o, l = _thd_call(cfg)
    ref_o, ref_l = attn_fwd_thd(x.q, x.k, x.v, x.sinks, x.cu_seqlens, cfg.softmax_scale, cfg.window,
                                rope_tables=_tables(cfg.rope))
    assert_parity(o, ref_o, cfg.name + " out (every element)")
    assert_lse_parity(l, ref_l, cfg.name + " lse (every element)")


def test_thd_full_context_full_size_every_element(cuda_device):
    cfg = THD_FULL
    x, o, l = _thd_call(cfg)
    ref_o, ref_l = attn_fwd_thd(x.q, x.k, x.v, x.sinks, x.cu_seqlens, cfg.softmax_scale, cfg.window,
                                rope_tables=_tables(cfg.rope))
    assert_parity(o, ref_o, cfg.name + " out (every element)")
    assert_lse_parity(l, ref_l, cfg.name + " lse (every element)")


@pytest.mark.parametrize("cfg", [DECODE_B64, DECODE_B64_W, DECODE_B8, DECODE_B8_W], ids=lambda c: c.name)
def test_decode_full_size_every_sequence(cuda_device, cfg):
    q, kc, vc, sinks, seqlens = make_decode_device(cfg, cuda_device)
    out, lse = ops.gptoss_attn_decode(q, kc, vc, seqlens, sinks, window=cfg.window,
                                      rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    tables = _tables(cfg.rope)
    qh, sh = host(q), host(sinks)
    lo = max(0, cfg.L - cfg.window) if cfg.window > 0 else 0
    ref_o = np.zeros(qh.shape)
    ref_l = np.zeros(qh.shape[:2])
    # the query rotated by the oracle at its true position L - 1; the decode
    # oracle then sees only the visible cache rows [lo, L), which travel to the
    # host one sequence at a time
    q_rot = rope(qh, np.full(cfg.B, cfg.L - 1), *tables)
    for b in range(cfg.B):
        ro, rl = attn_decode(q_rot[b:b + 1], host(kc[b:b + 1, lo:cfg.L]), host(vc[b:b + 1, lo:cfg.L]),
                             [cfg.L - lo], sh, 0.125, cfg.window)
        ref_o[b], ref_l[b] = ro[0], rl[0]
    assert_parity(host(out), ref_o, f"{cfg.name} out (every sequence)")
    assert_lse_parity(host(lse), ref_l, f"{cfg.name} lse (every sequence)")
