"""Device failure path without a GPU fault.

Every pipeline wait in the kernels is bounded; when one gives up the kernel
records GPTOSS_ERR_TIMEOUT in the device status word and returns.  Here a
wait on a barrier that nothing ever arrives at (the library's self test)
must time out after a short limit, the status must be readable and
resettable, and the CUDA context must stay usable for a normal call.
"""

import numpy as np
import pytest
import torch

from attention_yarn_rope_b200 import _abi, ops
from attention_yarn_rope_b200.workloads import PLAIN_ROPE, TINY, make_prefill
from oracle.attention import attn_fwd_bshd
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import assert_parity, dev, f32, host

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives(cuda_device):
    assert ops.read_device_status(reset=True) in (0, _abi.GPTOSS_ERR_TIMEOUT)
    res = torch.full((1,), 7, dtype=torch.int32, device=cuda_device)
    ops.selftest_wait_timeout(2000, res)  # 2 ms
    torch.cuda.synchronize()
    assert int(res.item()) == 0                      # the wait did not succeed ...
    assert ops.read_device_status(reset=True) == _abi.GPTOSS_ERR_TIMEOUT   # ... and said so
    assert ops.read_device_status(reset=True) == 0   # reset worked
    # the context is intact: a normal prefill still matches the oracle
    x = make_prefill(TINY)
    out = ops.gptoss_attn_fwd(dev(x.q), dev(x.k), dev(x.v), f32(x.sinks), rope=ops.RopeConfig.from_dict(PLAIN_ROPE))
    torch.cuda.synchronize()
    tabs = yarn_inv_freq_and_concentration(64, 150000.0, 1.0)
    ref, _ = attn_fwd_bshd(x.q, x.k, x.v, x.sinks, 0.125, 0, rope_tables=tabs)
    assert_parity(host(out), ref, "after timeout")
    assert ops.read_device_status(reset=False) == 0


def test_host_validation_raises(cuda_device):
    q = torch.zeros((1, 16, 8, 96), dtype=torch.bfloat16, device=cuda_device)  # head_dim 96 (64 and 128 only)
    with pytest.raises(_abi.GptossError) as e:
        ops.gptoss_attn_fwd(q, q[:, :, :1], q[:, :, :1], torch.zeros(8, device=cuda_device))
    assert e.value.status == _abi.GPTOSS_ERR_UNSUPPORTED
    q = torch.zeros((1, 16, 6, 64), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(_abi.GptossError) as e:
        ops.gptoss_attn_fwd(q, q[:, :, :4], q[:, :, :4], torch.zeros(6, device=cuda_device))  # 6 % 4 != 0
    assert e.value.status == _abi.GPTOSS_ERR_INVALID_ARG
