"""GPU parity of gptoss_attn_bwd against the float64 backward oracle.

Two kinds of check:
* kernel parity: both sides get the same stored forward output (the
  oracle's exact output rounded to bf16, as the API stores it) and lse; the
  oracle forms D = <dout, out> from that output, so the comparison isolates
  the backward's own arithmetic;
* end to end: the GPU forward's out / lse feed the GPU backward, compared
  with the exact gradient (D from the exact output).

Tolerance.  A gradient tensor has no fixed scale (dk sums over the query
heads of a group; dq / dk carry softmax_scale and the RoPE concentration),
so each is compared on its own unit scale, the RMS of the oracle's tensor,
the way the forward's outputs are: |got - ref| <= tol * max(RMS, |ref|)
element by element, and the mean error <= tol_mean * RMS.  The gradients are
heavy-tailed (the largest elements are 5-25 RMS), so their large elements
are held to a relative bound and the rest to the RMS.  The kernel's
roundings: rotated q / k as fp16, P as bf16 in P^T dout, dS as fp16 in the
products with q and k, fp32 accumulation, bf16 outputs (up to 2^-8
relative).  Exact arithmetic with only those roundings, emulated on the CPU
for the 2 x 300-row, 16-head case, gives at most 2.5e-2 (dv, from bf16 P;
dq / dk 4.6e-3) and means 0.9-1.7e-3 of the RMS, and the kernel measures the
same to within 15 %.  Bars (kernel parity): 5e-2 and 3e-3.  dsinks (fp32, an
atomic sum over rows): within 1e-2 of its RMS plus 1e-3.  End to end adds
the bf16 rounding of the stored output inside D = <dout, out>: dS = P (dP -
D) cancels where the sink share is small (dP ~ D), so a 2^-8 relative error
of D can become a much larger relative error of dS; measured at window 1
with N(0, 1) sinks: dq 9.1e-2 of the RMS at most, dk 3.5e-3 mean.  Bars
there: 1.5e-1 and 1e-2.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.attention import attn_fwd_bshd, attn_fwd_thd
from oracle.backward import attn_bwd_bshd, attn_bwd_thd
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import dev, f32, host, i32

pytestmark = pytest.mark.gpu

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)
SCALE = 0.125
MAX_REL = 5e-2
MEAN_REL = 3e-3


def assert_grad_parity(got, ref, what, max_rel=MAX_REL, mean_rel=MEAN_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert rms > 0, what
    err = np.abs(got - ref)
    scaled = err / np.maximum(rms, np.abs(ref))
    mx, mean = float(scaled.max()), float(err.mean()) / rms
    assert mx <= max_rel, f"{what}: scaled max error {mx:.3e} > {max_rel} (RMS {rms:.3e}, mean {mean:.3e} of it)"
    assert mean <= mean_rel, f"{what}: mean error {mean:.3e} of the RMS {rms:.3e} > {mean_rel}"
    return mx, mean


def assert_dsinks(got, ref, what):
    got = np.asarray(got, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(got - ref)
    assert np.all(err <= 1e-2 * rms + 1e-3), f"{what}: dsinks max error {err.max():.3e} (RMS {rms:.3e})"


def _inputs(rng, lead_q, lead_kv, Hq, Hkv):
    q = bf16_round(rng.standard_normal(lead_q + (Hq, 64)))
    k = bf16_round(rng.standard_normal(lead_kv + (Hkv, 64)))
    v = bf16_round(rng.standard_normal(lead_kv + (Hkv, 64)))
    dout = bf16_round(rng.standard_normal(lead_q + (Hq, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return q, k, v, dout, sinks


E2E_MAX_REL = 1.5e-1
E2E_MEAN_REL = 1e-2


def _oracle_fwd(q, k, v, sinks, window, tables, positions=None, cu=None):
    """The stored forward output (exact, rounded to bf16) and lse (fp32)."""
    if cu is None:
        out, lse = attn_fwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, window, rope_tables=tables,
                                 positions=positions)
    else:
        out, lse = attn_fwd_thd(q, k, v, sinks.astype(np.float64), cu, SCALE, window, rope_tables=tables,
                                positions=positions)
    return bf16_round(out), lse.astype(np.float32)


def _bwd(q, k, v, sinks, dout, out, lse, window, rope, **kw):
    """The GPU backward on host inputs; q, k, v may be given as device views."""
    qd = q if isinstance(q, torch.Tensor) else dev(q)
    kd = k if isinstance(k, torch.Tensor) else dev(k)
    vd = v if isinstance(v, torch.Tensor) else dev(v)
    dd = dout if isinstance(dout, torch.Tensor) else dev(dout)
    grads = ops.gptoss_attn_bwd(qd, kd, vd, f32(sinks), dev(out), dd, f32(lse), window=window, rope=rope, **kw)
    torch.cuda.synchronize()
    return grads


def _check_all(got, ref, what, max_rel=MAX_REL, mean_rel=MEAN_REL):
    dq, dk, dv, ds = got
    rq, rk, rv, rs = ref
    assert_grad_parity(host(dq), rq, f"{what} dq", max_rel, mean_rel)
    assert_grad_parity(host(dk), rk, f"{what} dk", max_rel, mean_rel)
    assert_grad_parity(host(dv), rv, f"{what} dv", max_rel, mean_rel)
    assert_dsinks(host(ds), rs, what)


@pytest.mark.parametrize("window", [0, 128, 1, 200])
def test_bwd_bshd_matches_oracle(cuda_device, window):
    # S = 300: four full 64-row tiles and a ragged one of 44
    rng = np.random.default_rng(101)
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    out, lse = _oracle_fwd(q, k, v, sinks, window, TABLES)
    got = _bwd(q, k, v, sinks, dout, out, lse, window, ROPE)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, window, dout, rope_tables=TABLES, out=out)
    _check_all(got, ref, f"bshd w={window}")


@pytest.mark.parametrize("explicit_positions", [False, True])
def test_bwd_thd_matches_oracle(cuda_device, explicit_positions):
    rng = np.random.default_rng(103)
    cu = np.array([0, 1, 78, 378, 378, 449], np.int64)  # lengths 1, 77, 300, 0, 71
    T, Hq, Hkv = int(cu[-1]), 16, 2
    q, k, v, dout, sinks = _inputs(rng, (T,), (T,), Hq, Hkv)
    pos = rng.integers(0, 131072 - 512, T).astype(np.int64) if explicit_positions else None
    out, lse = _oracle_fwd(q, k, v, sinks, 128, TABLES, positions=pos, cu=cu)
    kw = dict(cu_seqlens=i32(cu), max_seqlen=300)
    if pos is not None:
        kw["positions"] = i32(pos)
    got = _bwd(q, k, v, sinks, dout, out, lse, 128, ROPE, **kw)
    ref = attn_bwd_thd(q, k, v, sinks.astype(np.float64), cu, SCALE, 128, dout, rope_tables=TABLES, positions=pos,
                       out=out)
    _check_all(got, ref, f"thd positions={explicit_positions}")


def test_bwd_prerotated_inputs(cuda_device):
    # rope = None: q and k arrive rotated; the gradients are those of the
    # rotated inputs (no RoPE transpose)
    rng = np.random.default_rng(107)
    B, S, Hq, Hkv = 1, 200, 8, 1
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    out, lse = _oracle_fwd(q, k, v, sinks, 0, None)
    got = _bwd(q, k, v, sinks, dout, out, lse, 0, None)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, 0, dout, rope_tables=None, out=out)
    _check_all(got, ref, "pre-rotated")


def test_bwd_sink_minus_inf(cuda_device):
    rng = np.random.default_rng(109)
    B, S, Hq, Hkv = 1, 130, 8, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    sinks[0] = -np.inf
    sinks[5] = 30.0  # the sink takes nearly all the weight: small gradients everywhere but dsink
    out, lse = _oracle_fwd(q, k, v, sinks, 0, TABLES)
    got = _bwd(q, k, v, sinks, dout, out, lse, 0, ROPE)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, 0, dout, rope_tables=TABLES, out=out)
    assert host(got[3])[0] == 0.0
    _check_all(got, ref, "sinks -inf / +30")


def test_bwd_strided_views(cuda_device):
    # q, k, v as head slices of one fused [B, S, Hq + 2 Hkv, D] buffer; dout a
    # view with a padded head stride
    rng = np.random.default_rng(113)
    B, S, Hq, Hkv = 2, 150, 8, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    qkv = dev(np.concatenate([q, k, v], axis=2))
    dpad = torch.zeros((B, S, Hq + 3, 64), dtype=torch.bfloat16, device="cuda:0")
    dpad[:, :, :Hq] = dev(dout)
    out, lse = _oracle_fwd(q, k, v, sinks, 64, TABLES)
    got = _bwd(qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:], sinks, dpad[:, :, :Hq], out, lse, 64,
               ROPE)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, 64, dout, rope_tables=TABLES, out=out)
    _check_all(got, ref, "strided")


def test_bwd_no_rows(cuda_device):
    q = torch.empty((0, 64, 64), dtype=torch.bfloat16, device="cuda:0")
    k = torch.empty((0, 8, 64), dtype=torch.bfloat16, device="cuda:0")
    lse = torch.empty((64, 0), dtype=torch.float32, device="cuda:0")
    cu = i32([0, 0])
    ds = torch.full((64,), 7.0, device="cuda:0")
    ops.gptoss_attn_bwd(q, k, k, torch.zeros(64, device="cuda:0"), q, q, lse, rope=ROPE, cu_seqlens=cu,
                        max_seqlen=0, dsinks=ds)
    torch.cuda.synchronize()
    assert torch.all(ds == 0)


# Split sweeps: with G = 8 query heads per kv head, a key tile whose sweep
# covers more than 24 query tiles (more than 192 (head, tile) steps) is cut
# into chunks whose partial dK / dV add up in fp32 -- 1700 rows give key tile
# 0 twenty-seven query tiles (two chunks); window 1500 twenty-six.
@pytest.mark.parametrize("window", [0, 1500])
def test_bwd_split_sweeps(cuda_device, window):
    rng = np.random.default_rng(137)
    B, S, Hq, Hkv = 1, 1700, 16, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    out, lse = _oracle_fwd(q, k, v, sinks, window, TABLES)
    got = _bwd(q, k, v, sinks, dout, out, lse, window, ROPE)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, window, dout, rope_tables=TABLES, out=out)
    _check_all(got, ref, f"split sweeps w={window}")


def test_bwd_split_sweeps_thd(cuda_device):
    rng = np.random.default_rng(139)
    cu = np.array([0, 5, 1705, 1800], np.int64)  # lengths 5, 1700, 95
    T, Hq, Hkv = int(cu[-1]), 16, 2
    q, k, v, dout, sinks = _inputs(rng, (T,), (T,), Hq, Hkv)
    out, lse = _oracle_fwd(q, k, v, sinks, 0, TABLES, cu=cu)
    got = _bwd(q, k, v, sinks, dout, out, lse, 0, ROPE, cu_seqlens=i32(cu), max_seqlen=1700)
    ref = attn_bwd_thd(q, k, v, sinks.astype(np.float64), cu, SCALE, 0, dout, rope_tables=TABLES, out=out)
    _check_all(got, ref, "split sweeps thd")


def test_bwd_full_size_full_causal_slice(cuda_device):
    # the full-causal workload (B=2, S=8192, 64 / 8 heads): key tile 0 sweeps
    # 128 query tiles x 8 heads, cut into 6 chunks.  The GPU forward supplies
    # out / lse everywhere except the checked slice (batch row 1, kv group 2),
    # where the oracle's stored output and lse stand in; that slice's dq / dk /
    # dv depend on nothing else
    from attention_yarn_rope_b200.workloads import FULL, make_prefill

    x = make_prefill(FULL)
    dout = bf16_round(np.random.default_rng(149).standard_normal(x.q.shape, dtype=np.float32))
    b, g, G = 1, 2, 8
    heads = slice(g * G, (g + 1) * G)
    sinks = x.sinks.astype(np.float64)[heads]
    qs, ks, vs, ds_ = x.q[b:b + 1, :, heads], x.k[b:b + 1, :, g:g + 1], x.v[b:b + 1, :, g:g + 1], dout[b:b + 1, :, heads]
    o_sl, l_sl = _oracle_fwd(qs, ks, vs, x.sinks[heads], 0, TABLES)
    qd, kd, vd, sd = dev(x.q), dev(x.k), dev(x.v), f32(x.sinks)
    out, lse = ops.gptoss_attn_fwd(qd, kd, vd, sd, window=0, rope=ROPE, return_lse=True)
    out[b, :, heads] = dev(o_sl[0])
    lse[b, heads, :] = f32(l_sl[0])
    dq, dk, dv, _ = ops.gptoss_attn_bwd(qd, kd, vd, sd, out, dev(dout), lse, window=0, rope=ROPE)
    torch.cuda.synchronize()
    rq, rk, rv, _ = attn_bwd_bshd(qs, ks, vs, sinks, SCALE, 0, ds_, rope_tables=TABLES, out=o_sl)
    assert_grad_parity(host(dq[b:b + 1, :, heads]), rq, "full causal dq")
    assert_grad_parity(host(dk[b:b + 1, :, g:g + 1]), rk, "full causal dk")
    assert_grad_parity(host(dv[b:b + 1, :, g:g + 1]), rv, "full causal dv")


# Partial rotary (rotary_dim < 64): features [0, rotary_dim) rotate in pairs
# (j, j + rotary_dim / 2), the rest pass through without the concentration;
# the RoPE transpose in every backward epilogue follows.  W = 128 takes the
# mma.sync dQ kernel, W = 0 the tcgen05 one; 1700 rows split key tile 0's
# sweep (the finishing kernel's transpose).
@pytest.mark.parametrize("rotary_dim,window,S", [(32, 128, 300), (16, 0, 300), (48, 0, 1700), (48, 128, 300)])
def test_bwd_partial_rotary(cuda_device, rotary_dim, window, S):
    rng = np.random.default_rng(151)
    B, Hq, Hkv = 1, 16, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    tables = yarn_inv_freq_and_concentration(rotary_dim, 150000.0, 32.0, 4096, 1.0, 32.0)
    rope = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=rotary_dim)
    out, lse = _oracle_fwd(q, k, v, sinks, window, tables)
    got = _bwd(q, k, v, sinks, dout, out, lse, window, rope)
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, window, dout, rope_tables=tables, out=out)
    _check_all(got, ref, f"rotary_dim={rotary_dim} w={window} S={S}")


@pytest.mark.parametrize("window", [0, 1, 128])
def test_bwd_end_to_end(cuda_device, window):
    # GPU forward -> GPU backward against the exact gradient
    rng = np.random.default_rng(131)
    B, S, Hq, Hkv = 2, 300, 16, 2
    q, k, v, dout, sinks = _inputs(rng, (B, S), (B, S), Hq, Hkv)
    qd, kd, vd, sd = dev(q), dev(k), dev(v), f32(sinks)
    out, lse = ops.gptoss_attn_fwd(qd, kd, vd, sd, window=window, rope=ROPE, return_lse=True)
    got = ops.gptoss_attn_bwd(qd, kd, vd, sd, out, dev(dout), lse, window=window, rope=ROPE)
    torch.cuda.synchronize()
    ref = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), SCALE, window, dout, rope_tables=TABLES)
    _check_all(got, ref, f"end to end w={window}", E2E_MAX_REL, E2E_MEAN_REL)


def test_bwd_full_size_sliding_slice(cuda_device):
    # the benchmark's sliding workload (B=4, S=4096, 64 / 8 heads, W=128) run
    # whole on the GPU with the oracle's stored output; the oracle
    # differentiates one (batch row, kv group) slice -- its gradients depend on
    # nothing outside it -- and the sink gradient of that group's heads over
    # all four rows
    from attention_yarn_rope_b200.workloads import SLIDING, make_prefill

    x = make_prefill(SLIDING)
    dout = bf16_round(np.random.default_rng(127).standard_normal(x.q.shape, dtype=np.float32))
    out, lse = _oracle_fwd(x.q, x.k, x.v, x.sinks, 128, TABLES)
    dq, dk, dv, ds = _bwd(x.q, x.k, x.v, x.sinks, dout, out, lse, 128, ROPE)
    g, G = 5, 8
    heads = slice(g * G, (g + 1) * G)
    sinks = x.sinks.astype(np.float64)[heads]
    ds_ref = np.zeros(G)
    for b in range(4):
        rq, rk, rv, rs = attn_bwd_bshd(x.q[b:b + 1, :, heads], x.k[b:b + 1, :, g:g + 1], x.v[b:b + 1, :, g:g + 1],
                                       sinks, SCALE, 128, dout[b:b + 1, :, heads], rope_tables=TABLES,
                                       out=out[b:b + 1, :, heads])
        ds_ref += rs
        if b == 3:
            assert_grad_parity(host(dq[3:4, :, heads]), rq, "full-size dq")
            assert_grad_parity(host(dk[3:4, :, g:g + 1]), rk, "full-size dk")
            assert_grad_parity(host(dv[3:4, :, g:g + 1]), rv, "full-size dv")
    assert_dsinks(host(ds)[heads], ds_ref, "full-size")
