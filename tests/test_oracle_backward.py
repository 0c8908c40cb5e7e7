"""Pins of the backward oracle (oracle/backward.py) on the CPU.

Each check is independent of the chain-rule formulas the oracle writes out:
* central finite differences of ``L = sum(dout * out)`` through the forward
  oracle, coordinate by coordinate and along random directions (float64,
  truncation error ~eps^2);
* float64 ``torch.autograd`` of a forward restated here in PyTorch in another
  form (RoPE as a complex multiplication, the sink as an extra softmax column);
* the adjoint identity <rope(x), y> = <x, rope_transpose(y)>;
* the value-gradient row sums: sum_j dv_j = sum_i (1 - sink share_i) dout_i.
"""

import numpy as np
import pytest
import torch

from oracle.attention import attn_fwd_bshd, attn_fwd_thd
from oracle.backward import attn_bwd_bshd, attn_bwd_thd, rope_transpose
from oracle.rope import default_positions_bshd, rope
from oracle.yarn import yarn_inv_freq_and_concentration

TABLES = yarn_inv_freq_and_concentration(64, 150000.0, 32.0, 4096, 1.0, 32.0)
TABLES_PARTIAL = yarn_inv_freq_and_concentration(32, 150000.0, 32.0, 4096, 1.0, 32.0)  # rotary_dim 32
SCALE = 0.125


def _case(rng, B, S, Hq, Hkv, D=64):
    q = rng.standard_normal((B, S, Hq, D))
    k = rng.standard_normal((B, S, Hkv, D))
    v = rng.standard_normal((B, S, Hkv, D))
    sinks = rng.standard_normal(Hq)
    dout = rng.standard_normal((B, S, Hq, D))
    return q, k, v, sinks, dout


def _loss_bshd(q, k, v, sinks, dout, window, tables, positions=None):
    out, _ = attn_fwd_bshd(q, k, v, sinks, SCALE, window, rope_tables=tables, positions=positions)
    return float((out * dout).sum())


@pytest.mark.parametrize("window,tables", [(0, TABLES), (3, TABLES), (0, None), (2, None), (0, TABLES_PARTIAL)])
def test_finite_differences_bshd(window, tables):
    rng = np.random.default_rng(3)
    q, k, v, sinks, dout = _case(rng, 2, 6, 4, 2)
    dq, dk, dv, ds = attn_bwd_bshd(q, k, v, sinks, SCALE, window, dout, rope_tables=tables)
    eps = 1e-6
    args = [q, k, v, sinks]
    grads = [dq, dk, dv, ds]

    def loss(a):
        return _loss_bshd(a[0], a[1], a[2], a[3], dout, window, tables)

    # every sink, and 40 random coordinates of each tensor
    for ti, (x, gx) in enumerate(zip(args, grads)):
        idxs = list(np.ndindex(x.shape)) if x.ndim == 1 else [
            tuple(int(rng.integers(n)) for n in x.shape) for _ in range(40)]
        for idx in idxs:
            xp = [a.copy() for a in args]
            xm = [a.copy() for a in args]
            xp[ti][idx] += eps
            xm[ti][idx] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            assert abs(fd - gx[idx]) <= 1e-7 * max(1.0, abs(fd)), (ti, idx, fd, gx[idx])
    # three random directions through all inputs at once
    for _ in range(3):
        dirs = [rng.standard_normal(a.shape) for a in args]
        xp = [a + eps * d for a, d in zip(args, dirs)]
        xm = [a - eps * d for a, d in zip(args, dirs)]
        fd = (loss(xp) - loss(xm)) / (2 * eps)
        an = sum(float((g * d).sum()) for g, d in zip(grads, dirs))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd))


def test_finite_differences_thd_explicit_positions():
    rng = np.random.default_rng(5)
    cu = np.array([0, 3, 3, 8])  # an empty sequence in the middle
    T, Hq, Hkv = 8, 4, 1
    q = rng.standard_normal((T, Hq, 64))
    k = rng.standard_normal((T, Hkv, 64))
    v = rng.standard_normal((T, Hkv, 64))
    sinks = rng.standard_normal(Hq)
    dout = rng.standard_normal((T, Hq, 64))
    pos = rng.integers(0, 131072, T)
    dq, dk, dv, ds = attn_bwd_thd(q, k, v, sinks, cu, SCALE, 4, dout, rope_tables=TABLES, positions=pos)

    def loss(a):
        out, _ = attn_fwd_thd(a[0], a[1], a[2], a[3], cu, SCALE, 4, rope_tables=TABLES, positions=pos)
        return float((out * dout).sum())

    eps = 1e-6
    args = [q, k, v, sinks]
    for _ in range(4):
        dirs = [rng.standard_normal(a.shape) for a in args]
        fd = (loss([a + eps * d for a, d in zip(args, dirs)]) - loss([a - eps * d for a, d in zip(args, dirs)])) / (
            2 * eps)
        an = sum(float((g * d).sum()) for g, d in zip([dq, dk, dv, ds], dirs))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd))


def _torch_forward(q, k, v, sinks, window, inv_freq, conc, positions):
    """The forward restated in PyTorch: RoPE as a complex product on (x_i, x_{i+R}),
    the sink as one more column of a standard softmax (its value row is zero)."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    R = D // 2
    th = positions[..., None].to(torch.float64) * inv_freq  # [B, S, R]
    rot = torch.polar(torch.full_like(th, conc), th)[:, :, None, :]

    def rotate(x):
        z = torch.complex(x[..., :R], x[..., R:]) * rot
        return torch.cat([z.real, z.imag], dim=-1)

    qr, kr = rotate(q), rotate(k)
    kr = kr.repeat_interleave(Hq // Hkv, dim=2)
    vv = v.repeat_interleave(Hq // Hkv, dim=2)
    logits = torch.einsum("bihd,bjhd->bhij", qr, kr) * SCALE
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    allowed = j <= i
    if window > 0:
        allowed = allowed & (i - j < window)
    logits = logits.masked_fill(~allowed, float("-inf"))
    sink_col = sinks.view(1, Hq, 1, 1).expand(B, Hq, S, 1)
    w = torch.softmax(torch.cat([logits, sink_col], dim=-1), dim=-1)[..., :S]
    return torch.einsum("bhij,bjhd->bihd", w, vv)


@pytest.mark.parametrize("window", [0, 5])
def test_torch_autograd(window):
    rng = np.random.default_rng(7)
    q, k, v, sinks, dout = _case(rng, 2, 11, 8, 2)
    pos = default_positions_bshd(2, 11) + np.array([[0], [1000]])
    dq, dk, dv, ds = attn_bwd_bshd(q, k, v, sinks, SCALE, window, dout, rope_tables=TABLES, positions=pos)
    tq, tk, tv, ts = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, sinks))
    out = _torch_forward(tq, tk, tv, ts, window, torch.tensor(TABLES[0]), TABLES[1], torch.tensor(pos))
    (out * torch.tensor(dout)).sum().backward()
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (ds, ts.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("window", [0, 200])
def test_torch_autograd_several_row_blocks(window):
    # 1100 rows: three of the oracle's row blocks, key ranges cut by the window
    rng = np.random.default_rng(17)
    q, k, v, sinks, dout = _case(rng, 1, 1100, 2, 1)
    dq, dk, dv, ds = attn_bwd_bshd(q, k, v, sinks, SCALE, window, dout, rope_tables=TABLES)
    tq, tk, tv, ts = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, sinks))
    out = _torch_forward(tq, tk, tv, ts, window, torch.tensor(TABLES[0]), TABLES[1],
                         torch.tensor(default_positions_bshd(1, 1100)))
    (out * torch.tensor(dout)).sum().backward()
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (ds, ts.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-9, atol=1e-9)


def test_rope_transpose_is_the_adjoint():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 3, 64))
    y = rng.standard_normal((5, 3, 64))
    pos = rng.integers(0, 100000, 5)
    inv, c = TABLES
    lhs = float((rope(x, pos, inv, c) * y).sum())
    rhs = float((x * rope_transpose(y, pos, inv, c)).sum())
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))
    # and c^2 R^T R = c^2 I: the transpose undoes the rotation up to c^2
    np.testing.assert_allclose(rope_transpose(rope(x, pos, inv, c), pos, inv, c), c * c * x, rtol=0, atol=1e-12)


def test_rope_transpose_partial_rotary():
    # rotary_dim 32: pairs (j, j + 16) for j < 16 rotate; features 32..63 pass
    # through unchanged (no concentration) in both directions
    rng = np.random.default_rng(10)
    x = rng.standard_normal((5, 3, 64))
    y = rng.standard_normal((5, 3, 64))
    pos = rng.integers(0, 100000, 5)
    inv, c = TABLES_PARTIAL
    assert inv.shape == (16,)
    lhs = float((rope(x, pos, inv, c) * y).sum())
    rhs = float((x * rope_transpose(y, pos, inv, c)).sum())
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))
    np.testing.assert_array_equal(rope_transpose(y, pos, inv, c)[..., 32:], y[..., 32:])
    np.testing.assert_allclose(rope_transpose(rope(x, pos, inv, c), pos, inv, c)[..., :32], c * c * x[..., :32],
                               rtol=0, atol=1e-12)


def test_value_gradient_row_sums():
    rng = np.random.default_rng(11)
    q, k, v, sinks, dout = _case(rng, 1, 9, 4, 2)
    _, lse = attn_fwd_bshd(q, k, v, sinks, SCALE, 0, rope_tables=TABLES)
    _, _, dv, _ = attn_bwd_bshd(q, k, v, sinks, SCALE, 0, dout, rope_tables=TABLES)
    share = np.exp(sinks[None, :, None] - lse)  # [B, Hq, S]
    for g in range(2):
        heads = [2 * g, 2 * g + 1]
        want = sum(((1 - share[0, h])[:, None] * dout[0, :, h, :]).sum(axis=0) for h in heads)
        np.testing.assert_allclose(dv[0, :, g, :].sum(axis=0), want, rtol=0, atol=1e-12)


def test_sink_minus_inf_has_zero_gradient():
    rng = np.random.default_rng(13)
    q, k, v, sinks, dout = _case(rng, 1, 5, 2, 1)
    sinks[1] = -np.inf
    _, _, _, ds = attn_bwd_bshd(q, k, v, sinks, SCALE, 0, dout, rope_tables=TABLES)
    assert ds[1] == 0.0 and ds[0] != 0.0


def test_given_exact_output_changes_nothing():
    # D formed from the exact forward output equals D from the weights
    rng = np.random.default_rng(19)
    q, k, v, sinks, dout = _case(rng, 2, 40, 4, 2)
    out, _ = attn_fwd_bshd(q, k, v, sinks, SCALE, 7, rope_tables=TABLES)
    a = attn_bwd_bshd(q, k, v, sinks, SCALE, 7, dout, rope_tables=TABLES)
    b = attn_bwd_bshd(q, k, v, sinks, SCALE, 7, dout, rope_tables=TABLES, out=out)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)
    # a perturbed output moves D and, through dS, every gradient but dv
    c = attn_bwd_bshd(q, k, v, sinks, SCALE, 7, dout, rope_tables=TABLES, out=out * (1 + 1e-3))
    assert np.abs(c[0] - a[0]).max() > 1e-6 and np.array_equal(c[2], a[2])
