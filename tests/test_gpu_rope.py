"""GPU parity of gptoss_rope_qk against the float64 oracle.

The kernel reduces each angle in double precision and rotates in fp32, so
every output must sit within one bf16 spacing of the exact (float64) rotated
value -- a far tighter bar than the attention tolerance, and the check that
pins the angle precision at positions up to 131071.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import ops
from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, PLAIN_ROPE, bf16_round
from oracle.rope import default_positions_bshd, default_positions_thd, rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import bf16_ulp, dev, host, i32

pytestmark = pytest.mark.gpu


def _tables(rp):
    return yarn_inv_freq_and_concentration(64, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                           rp["ntk_beta"])


def _check(got, ref):
    err = np.abs(got - ref)
    assert np.all(err <= bf16_ulp(ref) + 1e-6), f"max err {err.max():.3e}"


@pytest.mark.parametrize("rp", [PLAIN_ROPE, GPTOSS_ROPE], ids=["plain", "yarn"])
@pytest.mark.parametrize("B,S,Hq,Hkv", [(1, 128, 8, 1), (2, 77, 64, 8), (1, 1, 4, 4)])
def test_rope_bshd(cuda_device, rp, B, S, Hq, Hkv):
    rng = np.random.default_rng(B * 1000 + S)
    q = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    k = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    qo, ko = ops.gptoss_rope_qk(dev(q), dev(k), ops.RopeConfig.from_dict(rp))
    torch.cuda.synchronize()
    inv, c = _tables(rp)
    pos = default_positions_bshd(B, S)
    _check(host(qo), rope(q, pos, inv, c))
    _check(host(ko), rope(k, pos, inv, c))


def test_rope_thd_and_explicit_positions(cuda_device):
    rng = np.random.default_rng(7)
    cu = np.array([0, 5, 5, 200, 333], np.int64)
    T = int(cu[-1])
    q = bf16_round(rng.standard_normal((T, 64, 64)))
    k = bf16_round(rng.standard_normal((T, 8, 64)))
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE)
    inv, c = _tables(GPTOSS_ROPE)
    qo, ko = ops.gptoss_rope_qk(dev(q), dev(k), cfg, cu_seqlens=i32(cu))
    torch.cuda.synchronize()
    pos = default_positions_thd(cu)
    _check(host(qo), rope(q, pos, inv, c))
    _check(host(ko), rope(k, pos, inv, c))
    # explicit positions up to the 128K context edge
    pos = rng.integers(0, 131072, size=T)
    pos[:4] = [131071, 131070, 0, 65536]
    qo, ko = ops.gptoss_rope_qk(dev(q), dev(k), cfg, positions=i32(pos), cu_seqlens=i32(cu))
    torch.cuda.synchronize()
    _check(host(qo), rope(q, pos, inv, c))
    _check(host(ko), rope(k, pos, inv, c))


def test_rope_strided_and_in_place(cuda_device):
    # q / k as views of a fused qkv buffer; k rotated in place, q into a new tensor
    rng = np.random.default_rng(9)
    B, S = 2, 40
    qkv = bf16_round(rng.standard_normal((B, S, 64 + 8 + 8, 64)))
    t = dev(qkv)
    q, k = t[:, :, :64], t[:, :, 64:72]
    cfg = ops.RopeConfig.from_dict(GPTOSS_ROPE)
    qo, ko = ops.gptoss_rope_qk(q, k, cfg, k_out=k)
    torch.cuda.synchronize()
    inv, c = _tables(GPTOSS_ROPE)
    pos = default_positions_bshd(B, S)
    _check(host(qo), rope(qkv[:, :, :64], pos, inv, c))
    _check(host(t[:, :, 64:72]), rope(qkv[:, :, 64:72], pos, inv, c))
    np.testing.assert_array_equal(host(t[:, :, 72:]), qkv[:, :, 72:])  # v untouched


@pytest.mark.parametrize("rotary_dim", [16, 32, 48])
@pytest.mark.parametrize("rp", [PLAIN_ROPE, GPTOSS_ROPE], ids=["plain", "yarn"])
def test_rope_partial_rotary(cuda_device, rp, rotary_dim):
    # partial_rotary_factor = rotary_dim / 64: the first rotary_dim features
    # rotate in pairs (j, j + rotary_dim / 2), the rest pass through untouched
    rng = np.random.default_rng(rotary_dim)
    B, S, Hq, Hkv = 2, 150, 8, 2
    q = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    k = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    qo, ko = ops.gptoss_rope_qk(dev(q), dev(k), ops.RopeConfig.from_dict(rp, rotary_dim=rotary_dim))
    torch.cuda.synchronize()
    inv, c = yarn_inv_freq_and_concentration(64, rp["base"], rp["factor"], rp["initial_context"], rp["ntk_alpha"],
                                             rp["ntk_beta"], partial_rotary_factor=rotary_dim / 64)
    assert len(inv) == rotary_dim // 2
    pos = default_positions_bshd(B, S)
    _check(host(qo), rope(q, pos, inv, c))
    _check(host(ko), rope(k, pos, inv, c))
    np.testing.assert_array_equal(host(qo)[..., rotary_dim:], q[..., rotary_dim:])
    np.testing.assert_array_equal(host(ko)[..., rotary_dim:], k[..., rotary_dim:])
