"""The parity bar is reachable by the kernels' number formats (CPU only).

Emulates the exact definition with only the roundings the prefill kernel
makes -- rotated q / k rounded to fp16 for QK^T, unnormalised P rounded to
bf16 for P V, the output rounded to bf16 -- and checks it against the float64
oracle with the same bar the GPU tests use (raw 1e-2 per element where
|ref| <= 4, plus half a bf16 spacing above 4; mean-abs <= 1e-3).  It also shows why the QK^T operands are fp16:
rounding them to bf16 instead breaks the bar at the YaRN concentration.
"""

import numpy as np

from attention_yarn_rope_b200.workloads import bf16_round
from oracle.attention import attn_fwd_bshd
from oracle.rope import default_positions_bshd, rope
from oracle.yarn import yarn_inv_freq_and_concentration
from tests.gpu_util import out_bar

TABS = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)


def _f16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)


def _emulate(q, k, v, sinks, window, round_qk):
    B, S, Hq, _ = q.shape
    G = Hq // k.shape[2]
    pos = default_positions_bshd(B, S)
    out = np.zeros(q.shape)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    vis = (j <= i) & ((window == 0) | (i - j < window))
    for b in range(B):
        qr = round_qk(rope(q[b], pos[b], *TABS))
        kr = round_qk(rope(k[b], pos[b], *TABS))
        for h in range(Hq):
            s = np.where(vis, 0.125 * qr[:, h] @ kr[:, h // G].T, -np.inf)
            m = np.maximum(sinks[h], s.max(1))
            e = np.exp(s - m[:, None])
            z = np.exp(sinks[h] - m) + e.sum(1)
            out[b, :, h] = (bf16_round(e).astype(np.float64) @ v[b][:, h // G]) / z[:, None]
    return bf16_round(out).astype(np.float64)


def _case():
    rng = np.random.default_rng(1)
    B, S, Hq, Hkv = 1, 200, 8, 1
    q = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    k = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    v = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return q, k, v, sinks


def _bar_used(got, ref):
    """Largest share of the per-element bar that an element uses."""
    return float((np.abs(got - ref) / out_bar(ref)).max())


def test_kernel_number_formats_meet_the_bar():
    q, k, v, sinks = _case()
    for window in (0, 128):
        ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=TABS)
        emu = _emulate(q, k, v, sinks, window, _f16)
        assert _bar_used(emu, ref) < 0.9
        assert np.abs(emu - ref)[np.abs(ref) <= 4].max() < 0.9e-2
        assert np.abs(emu - ref).mean() < 0.6e-3


def test_bf16_qk_operands_would_use_most_of_the_budget():
    q, k, v, sinks = _case()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, 0, rope_tables=TABS)
    e16 = np.abs(_emulate(q, k, v, sinks, 0, _f16) - ref).mean()
    eb16 = np.abs(_emulate(q, k, v, sinks, 0, lambda x: bf16_round(x).astype(np.float64)) - ref).mean()
    assert eb16 > 1.5 * e16
