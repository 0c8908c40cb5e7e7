"""Python binding of libgptoss_attn: the three entry points under the same
names, taking torch tensors.

PyTorch supplies device memory and the current CUDA stream; every step of the
computation runs in the library's CUDA kernels.  Functions raise
:class:`~attention_yarn_rope_b200._abi.GptossError` on any non-OK status, and
:func:`~attention_yarn_rope_b200._abi.load` raises when the library is
missing.  There is no CPU path.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi


@dataclass(frozen=True)
class RopeConfig:
    """YaRN parameters (RotaryEmbedding on the NeMo AutoModel gpt_oss.rope_utils page)."""

    base: float = 150000.0
    factor: float = 32.0
    initial_context: int = 4096
    ntk_alpha: float = 1.0
    ntk_beta: float = 32.0
    rotary_dim: int = 64

    def to_c(self) -> _abi.RopeParams:
        return _abi.RopeParams(float(self.base), float(self.factor), int(self.initial_context),
                               int(self.rotary_dim), float(self.ntk_alpha), float(self.ntk_beta))

    @staticmethod
    def from_dict(d: dict, rotary_dim: int = 64) -> "RopeConfig":
        return RopeConfig(d["base"], d["factor"], d["initial_context"], d["ntk_alpha"], d["ntk_beta"], rotary_dim)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _strides(t: torch.Tensor, thd: bool) -> _abi.Strides:
    if t.stride(-1) != 1:
        raise ValueError("head_dim must be contiguous")
    if thd:
        return _abi.Strides(0, t.stride(0), t.stride(1))
    return _abi.Strides(t.stride(0), t.stride(1), t.stride(2))


def _check_dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def gptoss_rope_qk(q, k, rope: RopeConfig, positions=None, cu_seqlens=None, q_out=None, k_out=None, stream=None):
    """YaRN RoPE of q ``[B,S,Hq,D]`` / ``[T,Hq,D]`` and k (Hkv heads).
    Returns ``(q_out, k_out)`` (new tensors unless given)."""
    lib = _abi.load()
    thd = cu_seqlens is not None
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    _check_dev(q, k, q_out, k_out, positions, cu_seqlens)
    if thd:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B, S_or_T = cu_seqlens.numel() - 1, T
    else:
        B, S_or_T, Hq, D = q.shape
        Hkv = k.shape[2]
    r = rope.to_c()
    st = lib.gptoss_rope_qk(_ptr(q), _strides(q, thd), _ptr(k), _strides(k, thd), _ptr(q_out),
                            _strides(q_out, thd), _ptr(k_out), _strides(k_out, thd), _ptr(positions),
                            _ptr(cu_seqlens), B, S_or_T, Hq, Hkv, D, ctypes.byref(r), _stream(stream))
    _abi.check("gptoss_rope_qk", st)
    return q_out, k_out


def gptoss_attn_fwd_workspace_size(total_tokens: int, Hkv: int, D: int = 64) -> int:
    return int(_abi.load().gptoss_attn_fwd_workspace_size(int(total_tokens), int(Hkv), int(D)))


def gptoss_attn_fwd(q, k, v, sinks, window: int = 0, softmax_scale: float | None = None,
                    rope: RopeConfig | None = None, positions=None, cu_seqlens=None, max_seqlen: int | None = None,
                    out=None, return_lse: bool = False, lse=None, workspace=None, stream=None):
    """Prefill sink attention.  BSHD when q is 4-D, packed THD when q is 3-D
    with ``cu_seqlens`` (then ``max_seqlen`` bounds the longest sequence).
    k (rotated when ``rope`` is given) and v are written once into a
    workspace as fp16 (``workspace``, or a new device buffer of
    ``gptoss_attn_fwd_workspace_size`` bytes).  Returns ``out`` or
    ``(out, lse)``."""
    lib = _abi.load()
    thd = cu_seqlens is not None
    out = torch.empty_like(q) if out is None else out
    if thd:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            if cu_seqlens.is_cuda:
                raise ValueError("max_seqlen is required when cu_seqlens lives on the device")
            max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max()) if B > 0 else 0
        S, total = int(max_seqlen), T
        lse_shape = (Hq, T)
    else:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        total = B * S
        lse_shape = (B, Hq, S)
    if return_lse and lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    _check_dev(q, k, v, sinks, out, lse, positions, cu_seqlens)
    scale = float(D) ** -0.5 if softmax_scale is None else float(softmax_scale)
    r = rope.to_c() if rope is not None else None
    if workspace is None:
        need = int(lib.gptoss_attn_fwd_workspace_size(total, Hkv, D))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_dev(workspace)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.gptoss_attn_fwd(_ptr(q), _strides(q, thd), _ptr(k), _strides(k, thd), _ptr(v), _strides(v, thd),
                             _ptr(sinks), _ptr(positions), _ptr(cu_seqlens), B, S, total, Hq, Hkv, D, int(window),
                             scale, ctypes.byref(r) if r is not None else None, _ptr(out), _strides(out, thd),
                             _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream))
    _abi.check("gptoss_attn_fwd", st)
    return (out, lse) if (return_lse or lse is not None) else out


def gptoss_attn_fwd_block_workspace_size(B: int, Sq: int, Sk: int, Hkv: int, D: int = 64) -> int:
    return int(_abi.load().gptoss_attn_fwd_block_workspace_size(int(B), int(Sq), int(Sk), int(Hkv), int(D)))


def gptoss_attn_fwd_block(q, k, v, q_start: int, k_start: int, softmax_scale: float | None = None,
                          rope: RopeConfig | None = None, out=None, lse=None, workspace=None, stream=None):
    """One key block of a query shard (context parallelism, full context):
    queries ``q [B,Sq,Hq,D]`` at global indices q_start.., keys / values
    ``[B,Sk,Hkv,D]`` at k_start.. (k_start <= q_start), causal on the global
    indices, no sink.  Returns ``(out fp32 [B,Sq,Hq,D], lse fp32 [B,Hq,Sq])``."""
    lib = _abi.load()
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if not (out.is_contiguous() and lse.is_contiguous()):
        raise ValueError("out and lse must be contiguous")
    if workspace is None:
        need = gptoss_attn_fwd_block_workspace_size(B, Sq, Sk, Hkv, D)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_dev(q, k, v, out, lse, workspace)
    scale = float(D) ** -0.5 if softmax_scale is None else float(softmax_scale)
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_attn_fwd_block(_ptr(q), _strides(q, False), _ptr(k), _strides(k, False), _ptr(v),
                                   _strides(v, False), B, Sq, Sk, int(q_start), int(k_start), Hq, Hkv, D, scale,
                                   ctypes.byref(r) if r is not None else None, _ptr(out), _ptr(lse),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _abi.check("gptoss_attn_fwd_block", st)
    return out, lse


def gptoss_attn_merge(outs, lses, sinks, out=None, lse=None, stream=None):
    """Merge block results of the same query rows and fold the sink in once:
    ``outs [n,B,S,Hq,D]`` fp32, ``lses [n,B,Hq,S]`` fp32, ``sinks [Hq]`` fp32
    (or None).  Returns ``out`` bf16 ``[B,S,Hq,D]`` or ``(out, lse)`` when
    ``lse`` is given or requested with ``lse=True``."""
    lib = _abi.load()
    n, B, S, Hq, D = outs.shape
    if not (outs.is_contiguous() and lses.is_contiguous()):
        raise ValueError("outs and lses must be contiguous")
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=outs.device)
    want_lse = lse is not None
    if lse is True:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=outs.device)
    _check_dev(outs, lses, sinks, out, lse if want_lse else None)
    st = lib.gptoss_attn_merge(_ptr(outs), _ptr(lses), n, _ptr(sinks), B, S, Hq, D, _ptr(out), _strides(out, False),
                               _ptr(lse) if want_lse else None, _stream(stream))
    _abi.check("gptoss_attn_merge", st)
    return (out, lse) if want_lse else out


def gptoss_qkv_rope_workspace_size(total_tokens: int, D: int = 64) -> int:
    return int(_abi.load().gptoss_qkv_rope_workspace_size(int(total_tokens), int(D)))


def gptoss_qkv_rope(x, w_qkv, b_qkv, Hq: int, Hkv: int, rope: RopeConfig | None = None, positions=None,
                    cu_seqlens=None, q_out=None, k_out=None, v_out=None, workspace=None, stream=None):
    """q, k, v projections of ``x`` (``[B,S,hidden]`` BSHD or ``[T,hidden]``
    with ``cu_seqlens``) through the stacked weights ``w_qkv [(Hq + 2 Hkv) D,
    hidden]`` and bias ``b_qkv`` (or None), q and k rotated when ``rope`` is
    given.  D = w_qkv.shape[0] // (Hq + 2 Hkv).  Returns ``(q, k, v)``."""
    lib = _abi.load()
    thd = cu_seqlens is not None
    N, hidden = w_qkv.shape
    D = N // (Hq + 2 * Hkv)
    if thd:
        T = x.shape[0]
        B, S_or_T = cu_seqlens.numel() - 1, T
        lead = (T,)
    else:
        B, S = x.shape[0], x.shape[1]
        S_or_T, T = S, B * S
        lead = (B, S)
    if x.shape[-1] != hidden or x.stride(-1) != 1:
        raise ValueError("x must be [..., hidden] with hidden contiguous")
    x_row_stride = x.stride(-2)
    if not thd and x.stride(0) != S * x_row_stride:
        raise ValueError("BSHD x must have uniform token rows")
    q_out = torch.empty(lead + (Hq, D), dtype=torch.bfloat16, device=x.device) if q_out is None else q_out
    k_out = torch.empty(lead + (Hkv, D), dtype=torch.bfloat16, device=x.device) if k_out is None else k_out
    v_out = torch.empty(lead + (Hkv, D), dtype=torch.bfloat16, device=x.device) if v_out is None else v_out
    if workspace is None and rope is not None:
        workspace = torch.empty(int(lib.gptoss_qkv_rope_workspace_size(T, D)), dtype=torch.uint8, device=x.device)
    _check_dev(x, w_qkv, b_qkv, positions, cu_seqlens, q_out, k_out, v_out, workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_qkv_rope(_ptr(x), int(x_row_stride), _ptr(w_qkv), _ptr(b_qkv), _ptr(positions),
                             _ptr(cu_seqlens), B, S_or_T, hidden, Hq, Hkv, D,
                             ctypes.byref(r) if r is not None else None, _ptr(q_out), _strides(q_out, thd),
                             _ptr(k_out), _strides(k_out, thd), _ptr(v_out), _strides(v_out, thd), _ptr(workspace),
                             ws_bytes, _stream(stream))
    _abi.check("gptoss_qkv_rope", st)
    return q_out, k_out, v_out


def gptoss_attn_bwd_workspace_size(total_tokens: int, Hq: int, Hkv: int, D: int = 64) -> int:
    return int(_abi.load().gptoss_attn_bwd_workspace_size(total_tokens, Hq, Hkv, D))


def gptoss_attn_bwd(q, k, v, sinks, out, dout, lse, window: int = 0, softmax_scale: float | None = None,
                    rope: RopeConfig | None = None, positions=None, cu_seqlens=None, max_seqlen: int | None = None,
                    dq=None, dk=None, dv=None, dsinks=None, workspace=None, stream=None):
    """Gradients of :func:`gptoss_attn_fwd` for ``L = sum(dout * out)``: q, k,
    v, sinks, window, scale, rope, positions and cu_seqlens exactly as given to
    the forward, ``out`` and ``lse`` from it.  Returns ``(dq, dk, dv, dsinks)``
    (dq / dk / dv bf16 contiguous in q / k / v's logical shapes, dsinks fp32)."""
    lib = _abi.load()
    thd = cu_seqlens is not None
    if thd:
        T, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            if cu_seqlens.is_cuda:
                raise ValueError("max_seqlen is required when cu_seqlens lives on the device")
            max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max()) if B > 0 else 0
        S, total = int(max_seqlen), T
    else:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        total = B * S
    dq = torch.empty(q.shape, dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=k.dtype, device=k.device) if dk is None else dk
    dv = torch.empty(v.shape, dtype=v.dtype, device=v.device) if dv is None else dv
    dsinks = torch.empty(Hq, dtype=torch.float32, device=q.device) if dsinks is None else dsinks
    for t in (dq, dk, dv, dsinks):
        if not t.is_contiguous():
            raise ValueError("gradient outputs must be contiguous")
    need = gptoss_attn_bwd_workspace_size(total, Hq, Hkv, D) if total > 0 else 0
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_dev(q, k, v, sinks, out, dout, lse, positions, cu_seqlens, dq, dk, dv, dsinks, workspace)
    scale = float(D) ** -0.5 if softmax_scale is None else float(softmax_scale)
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_attn_bwd(_ptr(q), _strides(q, thd), _ptr(k), _strides(k, thd), _ptr(v), _strides(v, thd),
                             _ptr(out), _strides(out, thd), _ptr(dout), _strides(dout, thd), _ptr(lse), _ptr(sinks),
                             _ptr(positions), _ptr(cu_seqlens), B, S, total, Hq, Hkv, D, int(window), scale,
                             ctypes.byref(r) if r is not None else None, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsinks),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _abi.check("gptoss_attn_bwd", st)
    return dq, dk, dv, dsinks


def gptoss_attn_decode_workspace_size(B: int, Lmax: int, Hq: int, Hkv: int, D: int = 64) -> int:
    return int(_abi.load().gptoss_attn_decode_workspace_size(B, Lmax, Hq, Hkv, D))


def gptoss_attn_decode(q, k_cache, v_cache, cache_seqlens, sinks, window: int = 0,
                       softmax_scale: float | None = None, rope: RopeConfig | None = None, out=None,
                       return_lse: bool = False, lse=None, workspace=None, stream=None):
    """Single-token decode: q ``[B,Hq,D]`` raw, caches ``[B,Lmax,Hkv,D]`` (keys
    rotated), ``cache_seqlens [B]`` int32 on the device."""
    lib = _abi.load()
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    out = torch.empty_like(q) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = gptoss_attn_decode_workspace_size(B, Lmax, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_dev(q, k_cache, v_cache, cache_seqlens, sinks, out, lse, workspace)
    for t in (q, k_cache, v_cache, out):
        if not t.is_contiguous():
            raise ValueError("decode tensors must be contiguous")
    scale = float(D) ** -0.5 if softmax_scale is None else float(softmax_scale)
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens), _ptr(sinks), B, Lmax,
                                Hq, Hkv, D, int(window), scale, ctypes.byref(r) if r is not None else None,
                                _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _abi.check("gptoss_attn_decode", st)
    return (out, lse) if (return_lse or lse is not None) else out


def gptoss_attn_decode_paged(q, k_pool, v_pool, block_table, cache_seqlens, sinks, window: int = 0,
                             softmax_scale: float | None = None, rope: RopeConfig | None = None, out=None,
                             return_lse: bool = False, lse=None, workspace=None, stream=None):
    """Decode over a paged cache: pools ``[num_blocks, block_size, Hkv, D]``
    (keys rotated), ``block_table [B, max_blocks]`` int32 and ``cache_seqlens
    [B]`` int32 on the device.  ``q`` is ``[B, Hq, D]`` (one new token per
    sequence) or ``[B, q_len, Hq, D]`` (q_len new tokens, already in the cache,
    each attending causally: token i sees ``cache_seqlens[b] - q_len + 1 + i``
    keys); ``out`` and ``lse`` take q's leading shape."""
    lib = _abi.load()
    if q.dim() == 3:
        B, Hq, D = q.shape
        q_len = 1
    else:
        B, q_len, Hq, D = q.shape
    num_blocks, block_size, Hkv, _ = k_pool.shape
    max_blocks = block_table.shape[1]
    out = torch.empty_like(q) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    need = gptoss_attn_decode_workspace_size(B * q_len, max_blocks * block_size, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_dev(q, k_pool, v_pool, block_table, cache_seqlens, sinks, out, lse, workspace)
    for t in (q, k_pool, v_pool, out, block_table):
        if not t.is_contiguous():
            raise ValueError("decode tensors must be contiguous")
    scale = float(D) ** -0.5 if softmax_scale is None else float(softmax_scale)
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_attn_decode_paged(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), max_blocks, block_size,
                                      num_blocks, _ptr(cache_seqlens), _ptr(sinks), B, q_len, Hq, Hkv, D, int(window),
                                      scale, ctypes.byref(r) if r is not None else None, _ptr(out), _ptr(lse),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _abi.check("gptoss_attn_decode_paged", st)
    return (out, lse) if (return_lse or lse is not None) else out


def gptoss_kv_append_paged(k_new, v_new, cache_seqlens, block_table, k_pool, v_pool, rope: RopeConfig | None,
                           stream=None):
    """Write each sequence's new tokens into the paged pools in place: ``k_new``,
    ``v_new`` ``[B, Hkv, D]`` (one token) or ``[B, q_len, Hkv, D]``; token i's key
    is rotated at position ``cache_seqlens[b] - q_len + i``."""
    lib = _abi.load()
    if k_new.dim() == 3:
        B, Hkv, D = k_new.shape
        q_len = 1
    else:
        B, q_len, Hkv, D = k_new.shape
    num_blocks, block_size = k_pool.shape[0], k_pool.shape[1]
    _check_dev(k_new, v_new, cache_seqlens, block_table, k_pool, v_pool)
    for t in (k_new, v_new, k_pool, v_pool, block_table):
        if not t.is_contiguous():
            raise ValueError("append tensors must be contiguous")
    r = rope.to_c() if rope is not None else None
    st = lib.gptoss_kv_append_paged(_ptr(k_new), _ptr(v_new), _ptr(cache_seqlens), _ptr(block_table),
                                    block_table.shape[1], block_size, _ptr(k_pool), _ptr(v_pool), num_blocks, B,
                                    q_len, Hkv, D, ctypes.byref(r) if r is not None else None, _stream(stream))
    _abi.check("gptoss_kv_append_paged", st)


def read_device_status(reset: bool = True, stream=None) -> int:
    v = ctypes.c_int32(0)
    _abi.check("gptoss_read_device_status",
               _abi.load().gptoss_read_device_status(ctypes.byref(v), 1 if reset else 0, _stream(stream)))
    return int(v.value)


def set_wait_limit(microseconds: int) -> None:
    _abi.check("gptoss_set_wait_limit", _abi.load().gptoss_set_wait_limit(int(microseconds)))


def selftest_wait_timeout(limit_us: int, result_dev: torch.Tensor, stream=None) -> None:
    _abi.check("gptoss_selftest_wait_timeout",
               _abi.load().gptoss_selftest_wait_timeout(int(limit_us), _ptr(result_dev), _stream(stream)))
