"""Context parallelism of the full-context layers on CPU (gloo ranks).

Each rank holds a contiguous shard of every sequence; the ring of
attention_yarn_rope_b200.cp.full_context_fwd must reproduce the unsharded
attention exactly.  The per-block attention and the merge are the float64
oracle's (oracle/cp.py), injected through the module's ``attn_block`` /
``merge`` arguments (the product defaults are the CUDA library), so these
tests check what the module adds -- the ring order, which blocks each rank
computes, the global offsets and RoPE positions, the merge inputs --
against the oracle of the whole sequence.
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
SEED = 29


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
    sinks = rng.standard_normal(HQ)
    return q, k, v, sinks


def _tables():
    from oracle.yarn import yarn_inv_freq_and_concentration

    return yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _oracle_block(q, k, v, q_start, k_start, rope=None, softmax_scale=None):
    """The oracle's block attention, batch row by batch row, RoPE at the global positions."""
    from oracle.cp import block_attention
    from oracle.rope import rope as rot

    scale = D ** -0.5 if softmax_scale is None else softmax_scale
    Sq, Sk = q.shape[1], k.shape[1]
    outs, lses = [], []
    for b in range(q.shape[0]):
        qr = rot(q[b].numpy(), np.arange(q_start, q_start + Sq), *rope)
        kr = rot(k[b].numpy(), np.arange(k_start, k_start + Sk), *rope)
        o, l = block_attention(qr, kr, v[b].numpy(), scale, 0, q_start, k_start)
        outs.append(o)
        lses.append(l)
    return torch.from_numpy(np.stack(outs)), torch.from_numpy(np.stack(lses))


def _oracle_merge(outs, lses, sinks):
    from oracle.cp import merge_blocks

    res = [merge_blocks([(outs[i, b].numpy(), lses[i, b].numpy()) for i in range(outs.shape[0])], sinks.numpy())
           for b in range(outs.shape[1])]
    return torch.from_numpy(np.stack([r[0] for r in res])), torch.from_numpy(np.stack([r[1] for r in res]))


def _worker(rank, world, port, s_loc, q_out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from attention_yarn_rope_b200 import cp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, sinks = (torch.from_numpy(x) for x in _inputs(world * s_loc))
        sl = slice(rank * s_loc, (rank + 1) * s_loc)
        out, lse = cp.full_context_fwd(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), sinks,
                                       _tables(), attn_block=_oracle_block, merge=_oracle_merge)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, s_loc):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, s_loc, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world,s_loc", [(2, 24), (3, 17)])
def test_ring_equals_whole_sequence(world, s_loc):
    from oracle.attention import attn_fwd_bshd

    q, k, v, sinks = _inputs(world * s_loc)
    out, lse = attn_fwd_bshd(q, k, v, sinks, D ** -0.5, 0, rope_tables=_tables())
    for rank, o, l in _run(world, s_loc):
        sl = slice(rank * s_loc, (rank + 1) * s_loc)
        np.testing.assert_allclose(o, out[:, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, lse[:, :, sl], rtol=0, atol=1e-12)


def test_one_rank_without_a_process_group():
    sys.path.insert(0, ROOT)
    from attention_yarn_rope_b200 import cp
    from oracle.attention import attn_fwd_bshd

    q, k, v, sinks = (torch.from_numpy(x) for x in _inputs(30))
    out, lse = cp.full_context_fwd(q, k, v, sinks, _tables(), attn_block=_oracle_block, merge=_oracle_merge)
    ref, ref_l = attn_fwd_bshd(q.numpy(), k.numpy(), v.numpy(), sinks.numpy(), D ** -0.5, 0, rope_tables=_tables())
    np.testing.assert_allclose(out.numpy(), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), ref_l, rtol=0, atol=1e-12)
