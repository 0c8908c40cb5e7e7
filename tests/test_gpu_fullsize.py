"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times, checked on sampled outputs the oracle computes one by one:

* sliding-window prefill B=4, S=4096, 64/8 heads, window 128, YaRN RoPE;
* full-context prefill B=2, S=8192;
* packed THD pair, 32768 tokens, full and window 128;
* decode B=64 x 32768 and B=8 x 131072, full and window 128 (caches drawn
  on the device, sampled sequences read back for the oracle).

Sampled rows always include the tile edges (first / last row of a tile, the
first and last token of a sequence) besides random ones.
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
from oracle.attention import attn_decode, attn_rows_bshd, attn_rows_thd
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_parity, dev, f32, host, i32

pytestmark = pytest.mark.gpu


def _tables(rp):
    return yarn_inv_freq_and_concentration(64, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                           rp["ntk_beta"])


def _rows_bshd(cfg, n, seed):
    rng = np.random.default_rng(seed)
    rows = [(0, 0, 0), (cfg.B - 1, cfg.Hq - 1, cfg.S - 1), (0, 5, 127), (cfg.B - 1, 9, 128), (0, 63, cfg.S // 2)]
    for _ in range(n):
        rows.append((int(rng.integers(cfg.B)), int(rng.integers(cfg.Hq)), int(rng.integers(cfg.S))))
    return rows


@pytest.mark.parametrize("cfg", [SLIDING, FULL], ids=lambda c: c.name)
def test_prefill_full_size_sampled(cuda_device, cfg):
    x = make_prefill(cfg)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=cfg.window,
                                   rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    rows = _rows_bshd(cfg, 48, 5)
    ref_o, ref_l = attn_rows_bshd(x.q, x.k, x.v, x.sinks, cfg.softmax_scale, cfg.window, rows,
                                  rope_tables=_tables(cfg.rope))
    o = host(out)
    l = host(lse)
    got_o = np.stack([o[b, i, h] for (b, h, i) in rows])
    got_l = np.array([l[b, h, i] for (b, h, i) in rows])
    assert_parity(got_o, ref_o, cfg.name + " out")
    assert_parity(got_l, ref_l, cfg.name + " lse")
    assert np.all(np.isfinite(o))


@pytest.mark.parametrize("cfg", [THD_FULL, THD_WINDOW], ids=lambda c: c.name)
def test_thd_full_size_sampled(cuda_device, cfg):
    x = make_prefill(cfg)
    cu = x.cu_seqlens
    lens = np.diff(cu)
    out, lse = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), window=cfg.window,
                                   cu_seqlens=i32(cu), max_seqlen=int(lens.max()),
                                   rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    T = int(cu[-1])
    rows = [(int(cu[s]), s % 64) for s in range(len(lens))] + [(int(cu[s + 1]) - 1, 7) for s in range(len(lens))]
    rows += [(int(rng.integers(T)), int(rng.integers(64))) for _ in range(40)]
    ref_o, ref_l = attn_rows_thd(x.q, x.k, x.v, x.sinks, cu, cfg.softmax_scale, cfg.window, rows,
                                 rope_tables=_tables(cfg.rope))
    o = host(out)
    l = host(lse)
    assert_parity(np.stack([o[t, h] for (t, h) in rows]), ref_o, cfg.name + " out")
    assert_parity(np.array([l[h, t] for (t, h) in rows]), ref_l, cfg.name + " lse")


@pytest.mark.parametrize("cfg", [DECODE_B64, DECODE_B64_W, DECODE_B8, DECODE_B8_W], ids=lambda c: c.name)
def test_decode_full_size_sampled(cuda_device, cfg):
    q, kc, vc, sinks, seqlens = make_decode_device(cfg, cuda_device)
    out, lse = ops.gptoss_attn_decode(q, kc, vc, seqlens, sinks, window=cfg.window,
                                      rope=ops.RopeConfig.from_dict(cfg.rope), return_lse=True)
    torch.cuda.synchronize()
    picks = sorted({0, cfg.B - 1, cfg.B // 2})
    for b in picks:
        ref_o, ref_l = attn_decode(host(q[b:b + 1]), host(kc[b:b + 1]), host(vc[b:b + 1]), [cfg.L], host(sinks),
                                   0.125, cfg.window, rope_tables=_tables(cfg.rope))
        assert_parity(host(out[b:b + 1]), ref_o, f"{cfg.name} b={b} out")
        assert_parity(host(lse[b:b + 1]), ref_l, f"{cfg.name} b={b} lse")
