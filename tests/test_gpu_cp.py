"""Context parallelism of the sliding-window layers on one GPU: the two ranks
of a 2-way split played in turn by one process through the module's
per-rank functions (the halo handed over by hand, so no rank waits on
another), the CUDA prefill and backward doing the attention.  The shards'
outputs, put together, must match the oracle of the whole sequence (the
forward's bars) and the gradients the exact ones (the backward's end-to-end
bars: the GPU forward's bf16 output feeds D)."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import cp, ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.attention import attn_fwd_bshd
from oracle.backward import attn_bwd_bshd
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host
from tests.test_gpu_attn_bwd import E2E_MAX_REL, E2E_MEAN_REL, assert_dsinks, assert_grad_parity

pytestmark = pytest.mark.gpu

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)


def test_two_shards_sliding_window(cuda_device):
    rng = np.random.default_rng(151)
    B, s_loc, Hq, Hkv, W = 1, 300, 16, 2, 128
    S = 2 * s_loc
    q = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    k = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    v = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    dout = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    sh = [slice(0, s_loc), slice(s_loc, S)]
    qd = [dev(q[:, s]) for s in sh]
    kd = [dev(k[:, s]) for s in sh]
    vd = [dev(v[:, s]) for s in sh]
    dd = [dev(dout[:, s]) for s in sh]
    sd = f32(sinks)
    halo = [None, cp.kv_tail(kd[0], vd[0], cp.halo_rows(W, s_loc, 2))]
    fwd = [cp.local_fwd(qd[r], kd[r], vd[r], sd, W, ROPE, r, halo[r]) for r in range(2)]
    bwd = [cp.local_bwd(qd[r], kd[r], vd[r], sd, fwd[r][0], dd[r], fwd[r][1], W, ROPE, r, halo[r]) for r in range(2)]
    cp.add_halo_grads(bwd[0][1], bwd[0][2], bwd[1][4])
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    ref_o, ref_l = attn_fwd_bshd(q, k, v, sinks, 0.125, W, rope_tables=TABLES)
    assert_parity(np.concatenate([host(f[0]) for f in fwd], axis=1), ref_o, "cp out")
    assert_lse_parity(np.concatenate([host(f[1]) for f in fwd], axis=2), ref_l, "cp lse")
    rq, rk, rv, rs = attn_bwd_bshd(q, k, v, sinks.astype(np.float64), 0.125, W, dout, rope_tables=TABLES)
    for i, (ref, name) in enumerate(((rq, "dq"), (rk, "dk"), (rv, "dv"))):
        got = np.concatenate([host(b[i]) for b in bwd], axis=1)
        assert_grad_parity(got, ref, f"cp {name}", E2E_MAX_REL, E2E_MEAN_REL)
    assert_dsinks(host(bwd[0][3]) + host(bwd[1][3]), rs, "cp")


def test_two_shards_packed_stream(cuda_device):
    # a packed stream of sequences 250, 210, 140 long split into two 300-token
    # shards: the middle sequence straddles the boundary
    from oracle.attention import attn_fwd_thd
    from oracle.backward import attn_bwd_thd

    rng = np.random.default_rng(157)
    cu = [0, 250, 460, 600]
    t_loc, Hq, Hkv, W = 300, 16, 2, 128
    T = 2 * t_loc
    q = bf16_round(rng.standard_normal((T, Hq, 64)))
    k = bf16_round(rng.standard_normal((T, Hkv, 64)))
    v = bf16_round(rng.standard_normal((T, Hkv, 64)))
    dout = bf16_round(rng.standard_normal((T, Hq, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    sh = [slice(0, t_loc), slice(t_loc, T)]
    qd, kd, vd, dd = ([dev(a[s]) for s in sh] for a in (q, k, v, dout))
    sd = f32(sinks)
    halo_n = cp.halo_rows(W, t_loc, 2)
    halo = [None, torch.cat([kd[0][t_loc - halo_n:], vd[0][t_loc - halo_n:]], dim=1)]
    fwd = [cp.local_fwd_thd(qd[r], kd[r], vd[r], sd, cu, W, ROPE, r, halo[r]) for r in range(2)]
    bwd = [cp.local_bwd_thd(qd[r], kd[r], vd[r], sd, fwd[r][0], dd[r], fwd[r][1], cu, W, ROPE, r, halo[r])
           for r in range(2)]
    cp.add_halo_grads(bwd[0][1].unsqueeze(0), bwd[0][2].unsqueeze(0), bwd[1][4].unsqueeze(0))
    torch.cuda.synchronize()
    assert ops.read_device_status() == 0
    ref_o, ref_l = attn_fwd_thd(q, k, v, sinks, np.array(cu), 0.125, W, rope_tables=TABLES)
    assert_parity(np.concatenate([host(f[0]) for f in fwd], axis=0), ref_o, "cp thd out")
    assert_lse_parity(np.concatenate([host(f[1]) for f in fwd], axis=1), ref_l, "cp thd lse")
    rq, rk, rv, rs = attn_bwd_thd(q, k, v, sinks.astype(np.float64), np.array(cu), 0.125, W, dout, rope_tables=TABLES)
    for i, (ref, name) in enumerate(((rq, "dq"), (rk, "dk"), (rv, "dv"))):
        got = np.concatenate([host(b[i]) for b in bwd], axis=0)
        assert_grad_parity(got, ref, f"cp thd {name}", E2E_MAX_REL, E2E_MEAN_REL)
    assert_dsinks(host(bwd[0][3]) + host(bwd[1][3]), rs, "cp thd")
