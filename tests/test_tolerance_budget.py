"""The parity bar is reachable by the kernels' number formats (CPU only).

Emulates the exact definition with only the roundings the prefill kernel
makes -- rotated q / k rounded to fp16 for QK^T, unnormalised P rounded to
fp16 for P V, the output rounded to bf16 -- and checks it against the float64
oracle with the bar the GPU tests use (raw 1e-2 per element where
|ref| <= 4, plus half a bf16 spacing above 4; mean-abs <= 1e-3).

The kernel takes P against a running base rather than the exact row maximum,
so which elements its P rounding hurts most is not the emulation's draw.  The
guarantee therefore rests on the sum of each rounding source's largest
output error over the case, which bounds any coincidence of them: with fp16
P that sum stays under 1e-2; with bf16 P (2^-9 relative instead of 2^-12) it
does not, because the bf16 output of a value in [2, 4) alone may round by
7.8e-3.  The QK^T operands are fp16 for the same reason: bf16 would use a
large part of the budget at the YaRN concentration (logits scaled by c^2).
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


def _b16(x):
    return bf16_round(x).astype(np.float64)


def _exact(x):
    return np.asarray(x, np.float64)


def _emulate(q, k, v, sinks, window, round_qk, round_p, round_out):
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
            out[b, :, h] = (round_p(e) @ v[b][:, h // G]) / z[:, None]
    return round_out(out)


def _case():
    rng = np.random.default_rng(1)
    B, S, Hq, Hkv = 2, 300, 16, 2
    q = bf16_round(rng.standard_normal((B, S, Hq, 64)))
    k = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    v = bf16_round(rng.standard_normal((B, S, Hkv, 64)))
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return q, k, v, sinks


def _max_err_where(emu, ref, mask):
    return float(np.abs(emu - ref)[mask].max())


def test_kernel_number_formats_meet_the_bar():
    q, k, v, sinks = _case()
    for window in (0, 128):
        ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, window, rope_tables=TABS)
        emu = _emulate(q, k, v, sinks, window, _f16, _f16, _b16)
        assert float((np.abs(emu - ref) / out_bar(ref)).max()) < 0.9
        assert np.abs(emu - ref).mean() < 0.6e-3


def test_worst_case_sum_of_rounding_sources():
    q, k, v, sinks = _case()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, 128, rope_tables=TABS)
    small = np.abs(ref) <= 4.0  # where the raw 1e-2 bar applies
    qk = _max_err_where(_emulate(q, k, v, sinks, 128, _f16, _exact, _exact), ref, small)
    p16 = _max_err_where(_emulate(q, k, v, sinks, 128, _exact, _f16, _exact), ref, small)
    pb16 = _max_err_where(_emulate(q, k, v, sinks, 128, _exact, _b16, _exact), ref, small)
    # the bf16 output format's own rounding where |ref| is in [2, 4): half of 2^-6
    out_round = 0.5 * 2.0 ** -6
    assert qk + p16 + out_round < 1e-2
    assert qk + pb16 + out_round > 1e-2
    assert pb16 > 4 * p16


def test_bf16_qk_operands_would_use_most_of_the_budget():
    q, k, v, sinks = _case()
    ref, _ = attn_fwd_bshd(q, k, v, sinks, 0.125, 0, rope_tables=TABS)
    e16 = np.abs(_emulate(q, k, v, sinks, 0, _f16, _f16, _b16) - ref).mean()
    eb16 = np.abs(_emulate(q, k, v, sinks, 0, _b16, _f16, _b16) - ref).mean()
    assert eb16 > 1.5 * e16
