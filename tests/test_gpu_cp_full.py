"""GPU parity of the full-context context-parallel pieces against the oracle:
gptoss_attn_fwd_block (a query shard against a key block at global offsets,
no sink) against oracle/cp.py's block_attention, gptoss_attn_merge against
merge_blocks, and both together -- one GPU playing the ranks of a split in
turn, every rank's blocks at or before its shard merged -- against the
unsharded prefill oracle.  The NCCL ring itself is checked with gloo ranks on
the CPU (tests/test_cp_full.py); every GPU call of this suite has one GPU."""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, bf16_round
from oracle.attention import attn_fwd_bshd
from oracle.cp import block_attention, merge_blocks
from oracle.rope import rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_lse_parity, assert_parity, dev, f32, host

pytestmark = pytest.mark.gpu

TABS = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
ROPE = ops.RopeConfig.from_dict(GPTOSS_ROPE)


def _rand(shape, seed):
    return bf16_round(np.random.default_rng(seed).standard_normal(shape))


def _oracle_block(q, k, v, q_start, k_start):
    outs, lses = [], []
    for b in range(q.shape[0]):
        qr = rope(q[b], np.arange(q_start, q_start + q.shape[1]), *TABS)
        kr = rope(k[b], np.arange(k_start, k_start + k.shape[1]), *TABS)
        o, l = block_attention(qr, kr, v[b], 0.125, 0, q_start, k_start)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("Sq,Sk,q_start,k_start", [(300, 300, 600, 600), (300, 300, 600, 300), (200, 333, 900, 0),
                                                   (129, 1, 129, 128), (256, 256, 131000, 130744)])
def test_block_matches_oracle(cuda_device, Sq, Sk, q_start, k_start):
    B, Hq, Hkv = 2, 16, 2
    q, k, v = _rand((B, Sq, Hq, 64), 1), _rand((B, Sk, Hkv, 64), 2), _rand((B, Sk, Hkv, 64), 3)
    out, lse = ops.gptoss_attn_fwd_block(dev(q), dev(k), dev(v), q_start, k_start, rope=ROPE)
    torch.cuda.synchronize()
    ref_o, ref_l = _oracle_block(q, k, v, q_start, k_start)
    # fp32 output: no bf16 rounding of its own, the same raw bar
    assert_parity(host(out), ref_o, f"block out {Sq}x{Sk} @ {q_start}/{k_start}")
    assert_lse_parity(host(lse), ref_l, f"block lse {Sq}x{Sk} @ {q_start}/{k_start}")


def test_block_rejects_a_later_block(cuda_device):
    q, k = dev(_rand((1, 64, 8, 64), 4)), dev(_rand((1, 64, 1, 64), 5))
    with pytest.raises(RuntimeError):
        ops.gptoss_attn_fwd_block(q, k, k, 0, 64, rope=ROPE)


def test_merge_matches_oracle(cuda_device):
    B, S, Hq, n = 2, 77, 8, 3
    rng = np.random.default_rng(6)
    outs = rng.standard_normal((n, B, S, Hq, 64)).astype(np.float32)
    lses = (3.0 * rng.standard_normal((n, B, Hq, S))).astype(np.float32)
    lses[1, 0, 2, :5] = -np.inf  # blocks some rows see no key of
    sinks = rng.standard_normal(Hq).astype(np.float32)
    sinks[3] = -np.inf
    out, lse = ops.gptoss_attn_merge(f32(outs), f32(lses), f32(sinks), lse=True)
    torch.cuda.synchronize()
    ref_o = np.zeros((B, S, Hq, 64))
    ref_l = np.zeros((B, Hq, S))
    for b in range(B):
        o, l = merge_blocks([(outs[i, b].astype(np.float64), lses[i, b].astype(np.float64)) for i in range(n)],
                            sinks.astype(np.float64))
        ref_o[b], ref_l[b] = o, l
    assert_parity(host(out), ref_o, "merge out")
    assert_lse_parity(host(lse), ref_l, "merge lse")


@pytest.mark.parametrize("world,s_loc", [(3, 200), (2, 384)])
def test_ranks_in_turn_equal_whole_sequence(cuda_device, world, s_loc):
    # one GPU plays every rank of the split: rank r's queries against the
    # blocks of ranks 0..r, merged with the sink once
    B, Hq, Hkv = 2, 16, 2
    S = world * s_loc
    q, k, v = _rand((B, S, Hq, 64), 7), _rand((B, S, Hkv, 64), 8), _rand((B, S, Hkv, 64), 9)
    sinks = np.random.default_rng(10).standard_normal(Hq).astype(np.float32)
    qd, kd, vd = dev(q), dev(k), dev(v)
    got_o, got_l = [], []
    for r in range(world):
        qs = qd[:, r * s_loc:(r + 1) * s_loc]
        parts = [ops.gptoss_attn_fwd_block(qs, kd[:, j * s_loc:(j + 1) * s_loc], vd[:, j * s_loc:(j + 1) * s_loc],
                                           r * s_loc, j * s_loc, rope=ROPE) for j in range(r + 1)]
        o, l = ops.gptoss_attn_merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
                                     f32(sinks), lse=True)
        got_o.append(o)
        got_l.append(l)
    torch.cuda.synchronize()
    ref_o, ref_l = attn_fwd_bshd(q, k, v, sinks, 0.125, 0, rope_tables=TABS)
    assert_parity(np.concatenate([host(o) for o in got_o], axis=1), ref_o, "cp full out")
    assert_lse_parity(np.concatenate([host(l) for l in got_l], axis=2), ref_l, "cp full lse")
