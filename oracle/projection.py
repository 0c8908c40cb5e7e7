"""q, k, v projections of the attention input with RoPE applied, float64.

Test infrastructure: the reference the CUDA path is checked against.  The
product never imports it.

Sources:

* blog page "gpt-oss-20b 模型结构" (the printed module tree of
  GptOssForCausalLM): every decoder layer's ``GptOssAttention`` holds
  ``q_proj = Linear(2880, 4096, bias=True)``, ``k_proj = Linear(2880, 512,
  bias=True)``, ``v_proj = Linear(2880, 512, bias=True)``; a PyTorch Linear
  computes ``y = x W^T + b`` with ``W`` of shape ``[out_features,
  in_features]``.
* NeMo AutoModel ``gpt_oss.layers`` page (``GptOssAttention``: ``head_dim``,
  ``num_attention_heads``, ``num_key_value_heads``): the projected q and k are
  viewed as ``[..., heads, head_dim]`` (4096 = 64 heads x 64, 512 = 8 x 64)
  and rotated (``gpt_oss.rope_utils`` page, ``apply_rotary_emb_qk``) before
  the attention; v is not rotated.

Reading (the pages leave the layout of the three weights open): the weights
are the three Linear matrices stacked row-wise, q rows first, then k, then v
(``[(Hq + 2 Hkv) D, hidden]``), and the biases likewise; head h of q is
output features ``[h D, (h + 1) D)``.
"""

from __future__ import annotations

import numpy as np

from .rope import rope


def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """``x [T, in] @ w[out, in]^T + b[out]`` in float64."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    return y if b is None else y + np.asarray(b, np.float64)


def qkv_rope(x, w_qkv, b_qkv, positions, Hq: int, Hkv: int, D: int, rope_tables=None):
    """Projections of ``x [T, hidden]`` through the stacked weights, split
    into q ``[T, Hq, D]``, k ``[T, Hkv, D]``, v ``[T, Hkv, D]``; q and k
    rotated at ``positions [T]`` when ``rope_tables = (inv_freq,
    concentration)`` is given."""
    T = x.shape[0]
    y = linear(x, w_qkv, b_qkv)
    q = y[:, : Hq * D].reshape(T, Hq, D)
    k = y[:, Hq * D: (Hq + Hkv) * D].reshape(T, Hkv, D)
    v = y[:, (Hq + Hkv) * D:].reshape(T, Hkv, D)
    if rope_tables is not None:
        q = rope(q, positions, *rope_tables)
        k = rope(k, positions, *rope_tables)
    return q, k, v
