"""Context parallelism of the sliding-window layers on CPU (gloo ranks).

Each rank holds a contiguous shard of the sequence; the halo exchange of
attention_yarn_rope_b200.cp must reproduce the unsharded attention and its
gradients exactly.  The per-rank attention here is the float64 oracle,
injected through the module's ``attn_fwd`` / ``attn_bwd`` arguments (the
product default is the CUDA library), so these tests check the sharding,
positions, halo exchange, gradient return and sink-gradient reduction --
everything the module adds -- against the oracle of the whole sequence.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, HQ, HKV, D = 2, 4, 2, 64
SEED = 23


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs(S):
    rng = np.random.default_rng(SEED)
    q = rng.standard_normal((B, S, HQ, D))
    k = rng.standard_normal((B, S, HKV, D))
    v = rng.standard_normal((B, S, HKV, D))
    dout = rng.standard_normal((B, S, HQ, D))
    sinks = rng.standard_normal(HQ)
    return q, k, v, dout, sinks


def _tables():
    from oracle.yarn import yarn_inv_freq_and_concentration

    return yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _oracle_fwd(q, k, v, sinks, window, rope, positions, softmax_scale=None, **_):
    from oracle.attention import attn_fwd_bshd

    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    out, lse = attn_fwd_bshd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), scale, window, rope_tables=rope,
                             positions=positions.numpy())
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_bwd(q, k, v, sinks, out, dout, lse, window, rope, positions, softmax_scale=None, **_):
    from oracle.backward import attn_bwd_bshd

    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    g = attn_bwd_bshd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), scale, window, dout.numpy(), rope_tables=rope,
                      positions=positions.numpy())
    return tuple(torch.from_numpy(x) for x in g)


def _worker(rank, world, port, s_loc, window, q_out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from attention_yarn_rope_b200 import cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, dout, sinks = (torch.from_numpy(x) for x in _inputs(world * s_loc))
        sl = slice(rank * s_loc, (rank + 1) * s_loc)
        qs, ks, vs, ds = q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), dout[:, sl].contiguous()
        rope = _tables()
        out, lse = cp.sliding_window_fwd(qs, ks, vs, sinks, window, rope, attn_fwd=_oracle_fwd)
        dq, dk, dv, dsinks = cp.sliding_window_bwd(qs, ks, vs, sinks, out, ds, lse, window, rope,
                                                   attn_bwd=_oracle_bwd)
        q_out.put((rank, out.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy(), dsinks.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, s_loc, window):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, s_loc, window, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world,s_loc,window", [(2, 40, 16), (3, 33, 33), (3, 20, 1)])
def test_sharded_sliding_window_equals_whole_sequence(world, s_loc, window):
    from oracle.attention import attn_fwd_bshd
    from oracle.backward import attn_bwd_bshd

    S = world * s_loc
    q, k, v, dout, sinks = _inputs(S)
    rope = _tables()
    out, lse = attn_fwd_bshd(q, k, v, sinks, D ** -0.5, window, rope_tables=rope)
    dq, dk, dv, dsinks = attn_bwd_bshd(q, k, v, sinks, D ** -0.5, window, dout, rope_tables=rope)
    res = _run(world, s_loc, window)
    for rank, o, l, gq, gk, gv, gs in res:
        sl = slice(rank * s_loc, (rank + 1) * s_loc)
        np.testing.assert_allclose(o, out[:, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, lse[:, :, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(gq, dq[:, sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gk, dk[:, sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gv, dv[:, sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gs, dsinks, rtol=1e-12, atol=1e-11)


def test_shard_shorter_than_the_halo_is_refused():
    from attention_yarn_rope_b200 import cp

    assert cp.halo_rows(16, 15, 2) == 15
    with pytest.raises(ValueError):
        cp.halo_rows(16, 14, 2)
    with pytest.raises(ValueError):
        cp.halo_rows(0, 100, 2)  # full-context layers are not covered
    assert cp.halo_rows(128, 1, 1) == 0  # one rank: no halo


def test_one_rank_without_a_process_group():
    # no process group: the module is one rank, no halo, global positions from 0
    from attention_yarn_rope_b200 import cp
    from oracle.attention import attn_fwd_bshd

    q, k, v, _, sinks = (torch.from_numpy(x) for x in _inputs(50))
    out, lse = cp.sliding_window_fwd(q, k, v, sinks, 16, _tables(), attn_fwd=_oracle_fwd)
    ref, ref_lse = attn_fwd_bshd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), D ** -0.5, 16, rope_tables=_tables())
    np.testing.assert_allclose(out.numpy(), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), ref_lse, rtol=0, atol=1e-12)


# ---- packed (THD) streams: sequences straddle the ranks ----
CU_THD = [0, 5, 30, 31, 60]  # lengths 5, 25, 1, 29


def _inputs_thd(T):
    rng = np.random.default_rng(SEED + 1)
    return (rng.standard_normal((T, HQ, D)), rng.standard_normal((T, HKV, D)), rng.standard_normal((T, HKV, D)),
            rng.standard_normal((T, HQ, D)), rng.standard_normal(HQ))


def _oracle_fwd_thd(q, k, v, sinks, window, rope, positions, cu_seqlens, softmax_scale=None, **_):
    from oracle.attention import attn_fwd_thd

    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    out, lse = attn_fwd_thd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), cu_seqlens.numpy(), scale, window,
                            rope_tables=rope, positions=positions.numpy())
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_bwd_thd(q, k, v, sinks, out, dout, lse, window, rope, positions, cu_seqlens, softmax_scale=None, **_):
    from oracle.backward import attn_bwd_thd

    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    g = attn_bwd_thd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), cu_seqlens.numpy(), scale, window,
                     dout.numpy(), rope_tables=rope, positions=positions.numpy())
    return tuple(torch.from_numpy(x) for x in g)


def _worker_thd(rank, world, port, t_loc, window, q_out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from attention_yarn_rope_b200 import cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, dout, sinks = (torch.from_numpy(x) for x in _inputs_thd(world * t_loc))
        sl = slice(rank * t_loc, (rank + 1) * t_loc)
        qs, ks, vs, ds = q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), dout[sl].contiguous()
        rope = _tables()
        out, lse = cp.sliding_window_fwd_thd(qs, ks, vs, sinks, CU_THD, window, rope, attn_fwd=_oracle_fwd_thd)
        dq, dk, dv, dsinks = cp.sliding_window_bwd_thd(qs, ks, vs, sinks, out, ds, lse, CU_THD, window, rope,
                                                       attn_bwd=_oracle_bwd_thd)
        q_out.put((rank, out.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy(), dsinks.numpy()))
    finally:
        dist.destroy_process_group()


def test_sharded_packed_stream_equals_whole_stream():
    from oracle.attention import attn_fwd_thd
    from oracle.backward import attn_bwd_thd

    world, t_loc, window = 3, 20, 8
    q, k, v, dout, sinks = _inputs_thd(world * t_loc)
    rope = _tables()
    cu = np.array(CU_THD)
    out, lse = attn_fwd_thd(q, k, v, sinks, cu, D ** -0.5, window, rope_tables=rope)
    dq, dk, dv, dsinks = attn_bwd_thd(q, k, v, sinks, cu, D ** -0.5, window, dout, rope_tables=rope)
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_thd, args=(r, world, port, t_loc, window, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, o, l, gq, gk, gv, gs in res:
        sl = slice(rank * t_loc, (rank + 1) * t_loc)
        np.testing.assert_allclose(o, out[sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, lse[:, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(gq, dq[sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gk, dk[sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gv, dv[sl], rtol=0, atol=1e-11)
        np.testing.assert_allclose(gs, dsinks, rtol=1e-12, atol=1e-11)


def test_thd_local_layout():
    from attention_yarn_rope_b200.cp import thd_local_layout

    cu_l, pos, start = thd_local_layout(CU_THD, 1, 20, 7)  # extended stream = global tokens [13, 40)
    assert start == 13
    assert cu_l.tolist() == [0, 17, 18, 27]
    assert pos.tolist() == list(range(8, 25)) + [0] + list(range(0, 9))
    cu_l, pos, start = thd_local_layout(CU_THD, 0, 20, 7)  # rank 0: no halo
    assert (start, cu_l.tolist()) == (0, [0, 5, 20])
    with pytest.raises(ValueError):
        thd_local_layout(CU_THD, 2, 25, 7)  # shards past the stream's end
