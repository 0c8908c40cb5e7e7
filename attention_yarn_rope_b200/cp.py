"""Context parallelism for the sliding-window layers: one sequence split
along its length over the ranks of a process group.

The NeMo AutoModel gpt_oss.rope_utils page gives ``apply_rotary_emb_qk``
``cp_size`` / ``cp_rank`` arguments, with the local context-parallel shard in
the leading dimensions of q and k; it does not give the shards' layout.
Here rank r of R holds the contiguous tokens [r S_loc, (r + 1) S_loc) of
every sequence (BSHD ``[B, S_loc, H, D]``), so RoPE takes the global position
r S_loc + i.

GPT-OSS alternates full-context and 128-token sliding-window layers
(Transformers v4.55.0 release notes, "Architecture").  With a window of W
keys, query row i sees keys [i - W + 1, i]: the rows of rank r reach into
rank r - 1 by at most W - 1 keys, and no further while S_loc >= W - 1.  So
the forward needs one exchange -- rank r - 1 sends its last W - 1 rows of k
and v to rank r (a halo) -- after which rank r runs the ordinary prefill on
[halo | shard] with the halo's query rows left zero and their outputs
dropped.  Every query row of the shard then sees exactly its keys, the sink
once, so the result is the unsharded attention's, not an approximation.
The backward runs the ordinary backward on the same extended sequence with
zero dout for the halo rows (they contribute nothing), sends the halo rows'
dk / dv back to rank r - 1, which adds them to its last W - 1 rows, and sums
dsinks over the ranks.

Full-context layers need every earlier shard's keys: :func:`full_context_fwd`
passes the k / v shards around the ring of ranks (NCCL point-to-point, the
next block's transfer overlapping the current block's attention); each rank
runs the block form of the prefill (``gptoss_attn_fwd_block``: causal on the
global token indices, no sink) of its query shard against every block at or
before it, and merges the blocks with the sink folded in once
(``gptoss_attn_merge``).  Forward only.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops


def _rank_world(group):
    """(rank, world size) in `group`; one rank when no process group exists."""
    if not dist.is_available() or not dist.is_initialized():
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def _peer(group, rank: int) -> int:
    """Global rank of `rank` within `group` (point-to-point calls take global ranks)."""
    return rank if group is None else dist.get_global_rank(group, rank)


def _exchange(send_next, recv_shape, dtype, device, group, rank, world):
    """Send `send_next` to rank + 1 and receive a `recv_shape` tensor from rank - 1
    (None on rank 0).  Receives are posted before sends, so no rank blocks."""
    reqs = []
    recv = None
    if rank > 0:
        recv = torch.empty(recv_shape, dtype=dtype, device=device)
        reqs.append(dist.irecv(recv, src=_peer(group, rank - 1), group=group))
    send = send_next.contiguous() if rank + 1 < world else None  # alive until the send completes
    if send is not None:
        reqs.append(dist.isend(send, dst=_peer(group, rank + 1), group=group))
    for r in reqs:
        r.wait()
    return recv


def _exchange_back(send_prev, recv_shape, dtype, device, group, rank, world):
    """Send `send_prev` to rank - 1 and receive a `recv_shape` tensor from rank + 1
    (None on the last rank)."""
    reqs = []
    recv = None
    if rank + 1 < world:
        recv = torch.empty(recv_shape, dtype=dtype, device=device)
        reqs.append(dist.irecv(recv, src=_peer(group, rank + 1), group=group))
    send = send_prev.contiguous() if rank > 0 else None  # alive until the send completes
    if send is not None:
        reqs.append(dist.isend(send, dst=_peer(group, rank - 1), group=group))
    for r in reqs:
        r.wait()
    return recv


def halo_rows(window: int, s_loc: int, world: int) -> int:
    """Rows of k / v a rank needs from its predecessor: window - 1 (none on one rank)."""
    if window <= 0:
        raise ValueError("context parallelism here covers the sliding-window layers (window > 0)")
    halo = window - 1 if world > 1 else 0
    if s_loc < halo:
        raise ValueError(f"each shard needs at least window - 1 = {halo} tokens, got {s_loc}")
    return halo


def _positions(B: int, start: int, length: int, device) -> torch.Tensor:
    pos = torch.arange(start, start + length, dtype=torch.int32, device=device)
    return pos.unsqueeze(0).expand(B, length).contiguous()


def kv_tail(k, v, halo: int):
    """The last `halo` rows of this shard's k and v, heads concatenated: what
    the next rank receives."""
    s_loc = k.shape[1]
    return torch.cat([k[:, s_loc - halo:], v[:, s_loc - halo:]], dim=2)


def local_fwd(q, k, v, sinks, window: int, rope, rank: int, halo_kv=None, softmax_scale=None, attn_fwd=None):
    """Rank `rank`'s rows given `halo_kv` (the previous rank's :func:`kv_tail`,
    None on rank 0): the prefill over [halo | shard] at global positions,
    the halo's query rows zero and dropped.  No communication."""
    attn_fwd = attn_fwd or (lambda *a, **kw: ops.gptoss_attn_fwd(*a, return_lse=True, **kw))
    B, s_loc, Hq, D = q.shape
    Hkv = k.shape[2]
    if halo_kv is None:
        pos = _positions(B, rank * s_loc, s_loc, q.device)
        return attn_fwd(q, k, v, sinks, window=window, rope=rope, positions=pos, softmax_scale=softmax_scale)
    halo = halo_kv.shape[1]
    q_ext = torch.cat([torch.zeros((B, halo, Hq, D), dtype=q.dtype, device=q.device), q], dim=1)
    k_ext = torch.cat([halo_kv[:, :, :Hkv], k], dim=1)
    v_ext = torch.cat([halo_kv[:, :, Hkv:], v], dim=1)
    pos = _positions(B, rank * s_loc - halo, halo + s_loc, q.device)
    out, lse = attn_fwd(q_ext, k_ext, v_ext, sinks, window=window, rope=rope, positions=pos,
                        softmax_scale=softmax_scale)
    return out[:, halo:].contiguous(), lse[:, :, halo:].contiguous()


def local_bwd(q, k, v, sinks, out, dout, lse, window: int, rope, rank: int, halo_kv=None, softmax_scale=None,
              attn_bwd=None):
    """Rank `rank`'s gradients given `halo_kv`: ``(dq, dk, dv, dsinks, dkv_halo)``
    with dk / dv of its own rows (before the next rank's halo gradients are
    added), its share of dsinks, and the halo rows' dk / dv (heads
    concatenated, None on rank 0) that belong to the previous rank.  No
    communication."""
    attn_bwd = attn_bwd or ops.gptoss_attn_bwd
    B, s_loc, Hq, D = q.shape
    Hkv = k.shape[2]
    if halo_kv is None:
        pos = _positions(B, rank * s_loc, s_loc, q.device)
        dq, dk, dv, dsinks = attn_bwd(q, k, v, sinks, out, dout, lse, window=window, rope=rope, positions=pos,
                                      softmax_scale=softmax_scale)
        return dq, dk, dv, dsinks, None
    halo = halo_kv.shape[1]
    zq = torch.zeros((B, halo, Hq, D), dtype=q.dtype, device=q.device)
    q_ext = torch.cat([zq, q], dim=1)
    k_ext = torch.cat([halo_kv[:, :, :Hkv], k], dim=1)
    v_ext = torch.cat([halo_kv[:, :, Hkv:], v], dim=1)
    out_ext = torch.cat([zq, out], dim=1)
    dout_ext = torch.cat([zq, dout], dim=1)  # the halo rows are not this rank's: no gradient flows in
    # lse = +inf gives the halo rows zero weights (and zero sink share)
    lse_ext = torch.cat([torch.full((B, Hq, halo), float("inf"), dtype=lse.dtype, device=lse.device), lse], dim=2)
    pos = _positions(B, rank * s_loc - halo, halo + s_loc, q.device)
    dq_e, dk_e, dv_e, dsinks = attn_bwd(q_ext, k_ext, v_ext, sinks, out_ext, dout_ext, lse_ext, window=window,
                                        rope=rope, positions=pos, softmax_scale=softmax_scale)
    return (dq_e[:, halo:].contiguous(), dk_e[:, halo:].contiguous(), dv_e[:, halo:].contiguous(), dsinks,
            torch.cat([dk_e[:, :halo], dv_e[:, :halo]], dim=2))


def add_halo_grads(dk, dv, back):
    """Add the next rank's halo gradients `back` (heads concatenated) to the
    last rows of dk / dv, summed in fp32 at least and rounded once."""
    Hkv, halo, s_loc = dk.shape[2], back.shape[1], dk.shape[1]
    tail = slice(s_loc - halo, s_loc)
    acc = torch.promote_types(dk.dtype, torch.float32)
    dk[:, tail] = (dk[:, tail].to(acc) + back[:, :, :Hkv].to(acc)).to(dk.dtype)
    dv[:, tail] = (dv[:, tail].to(acc) + back[:, :, Hkv:].to(acc)).to(dv.dtype)


def sliding_window_fwd(q, k, v, sinks, window: int, rope, group=None, softmax_scale: float | None = None,
                       attn_fwd=None):
    """This rank's rows of the sliding-window attention of the whole sequence.

    q ``[B, S_loc, Hq, D]``, k / v ``[B, S_loc, Hkv, D]``: this rank's shard.
    Returns ``(out [B, S_loc, Hq, D], lse [B, Hq, S_loc])``.  ``attn_fwd``
    (keyword-compatible with :func:`ops.gptoss_attn_fwd`, returning
    ``(out, lse)``) defaults to the CUDA prefill."""
    rank, world = _rank_world(group)
    B, s_loc, _, D = q.shape
    Hkv = k.shape[2]
    halo = halo_rows(window, s_loc, world)
    got = None
    if halo:
        got = _exchange(kv_tail(k, v, halo), (B, halo, 2 * Hkv, D), k.dtype, k.device, group, rank, world)
    return local_fwd(q, k, v, sinks, window, rope, rank, got, softmax_scale, attn_fwd)


def sliding_window_bwd(q, k, v, sinks, out, dout, lse, window: int, rope, group=None,
                       softmax_scale: float | None = None, attn_bwd=None):
    """Gradients of this rank's shard for ``L = sum over all ranks of sum(dout * out)``.

    q, k, v, sinks, window, rope as given to :func:`sliding_window_fwd`; out,
    lse from it; dout this rank's ``[B, S_loc, Hq, D]``.  Returns ``(dq, dk,
    dv, dsinks)`` for this rank's tokens, dsinks summed over the group.
    ``attn_bwd`` (keyword-compatible with :func:`ops.gptoss_attn_bwd`)
    defaults to the CUDA backward."""
    rank, world = _rank_world(group)
    B, s_loc, _, D = q.shape
    Hkv = k.shape[2]
    halo = halo_rows(window, s_loc, world)
    got = None
    if halo:
        got = _exchange(kv_tail(k, v, halo), (B, halo, 2 * Hkv, D), k.dtype, k.device, group, rank, world)
    dq, dk, dv, dsinks, dkv_halo = local_bwd(q, k, v, sinks, out, dout, lse, window, rope, rank, got,
                                             softmax_scale, attn_bwd)
    if halo:  # the halo rows' key / value gradients belong to the previous rank's last rows
        back = _exchange_back(dkv_halo, (B, halo, 2 * Hkv, D), dk.dtype, dk.device, group, rank, world)
        if back is not None:
            add_halo_grads(dk, dv, back)
    dsinks = dsinks.clone()
    if world > 1:
        dist.all_reduce(dsinks, op=dist.ReduceOp.SUM, group=group)
    return dq, dk, dv, dsinks


# ----------------------------------------------------------------------------
# Packed (THD) inputs: rank r holds the contiguous tokens [r T_loc, (r + 1)
# T_loc) of the packed stream, whose sequences may straddle the ranks.  The
# extended stream [halo | shard] is re-packed with the global sequence
# boundaries cut to it; positions restart at every sequence start, as in the
# whole stream.  Halo tokens of a sequence that ends before the shard form
# their own local sequence; their outputs are dropped like every halo row's.
# ----------------------------------------------------------------------------
def thd_local_layout(cu_seqlens, rank: int, t_loc: int, halo: int):
    """Host-side layout of rank `rank`'s extended stream: ``(cu_local,
    positions, start)`` -- the local sequence boundaries (int32, from 0), each
    extended token's position inside its sequence (int32) and the global
    index of the first extended token.  `cu_seqlens` is the global packing
    (host integers)."""
    cu = [int(x) for x in cu_seqlens]
    start = rank * t_loc - (halo if rank > 0 else 0)
    end = (rank + 1) * t_loc
    if start < 0 or end > cu[-1]:
        raise ValueError("the shards must tile the packed stream exactly")
    bounds = [start] + [c for c in cu if start < c < end] + [end]
    cu_local = [b - start for b in bounds]
    pos = []
    s = 0
    for g in range(start, end):
        while cu[s + 1] <= g:
            s += 1
        pos.append(g - cu[s])
    return (torch.tensor(cu_local, dtype=torch.int32), torch.tensor(pos, dtype=torch.int32), start)


def _thd_ext(x, halo_x, halo: int):
    return x if halo_x is None else torch.cat([halo_x, x], dim=0)


def local_fwd_thd(q, k, v, sinks, cu_seqlens, window: int, rope, rank: int, halo_kv=None, softmax_scale=None,
                  attn_fwd=None):
    """THD form of :func:`local_fwd`: q ``[T_loc, Hq, D]``, k / v ``[T_loc,
    Hkv, D]``, `cu_seqlens` the global packing (host).  Returns ``(out
    [T_loc, Hq, D], lse [Hq, T_loc])``.  No communication."""
    attn_fwd = attn_fwd or (lambda *a, **kw: ops.gptoss_attn_fwd(*a, return_lse=True, **kw))
    t_loc, Hq, D = q.shape
    Hkv = k.shape[1]
    halo = 0 if halo_kv is None else halo_kv.shape[0]
    cu_l, pos, _ = thd_local_layout(cu_seqlens, rank, t_loc, halo)
    q_ext = _thd_ext(q, torch.zeros((halo, Hq, D), dtype=q.dtype, device=q.device) if halo else None, halo)
    k_ext = _thd_ext(k, halo_kv[:, :Hkv] if halo else None, halo)
    v_ext = _thd_ext(v, halo_kv[:, Hkv:] if halo else None, halo)
    max_len = int((cu_l[1:] - cu_l[:-1]).max())
    out, lse = attn_fwd(q_ext, k_ext, v_ext, sinks, window=window, rope=rope, positions=pos.to(q.device),
                        cu_seqlens=cu_l.to(q.device), max_seqlen=max_len, softmax_scale=softmax_scale)
    return out[halo:].contiguous(), lse[:, halo:].contiguous()


def local_bwd_thd(q, k, v, sinks, out, dout, lse, cu_seqlens, window: int, rope, rank: int, halo_kv=None,
                  softmax_scale=None, attn_bwd=None):
    """THD form of :func:`local_bwd`; returns ``(dq, dk, dv, dsinks,
    dkv_halo)`` with dkv_halo ``[halo, 2 Hkv, D]`` (None on rank 0)."""
    attn_bwd = attn_bwd or ops.gptoss_attn_bwd
    t_loc, Hq, D = q.shape
    Hkv = k.shape[1]
    halo = 0 if halo_kv is None else halo_kv.shape[0]
    cu_l, pos, _ = thd_local_layout(cu_seqlens, rank, t_loc, halo)
    zq = torch.zeros((halo, Hq, D), dtype=q.dtype, device=q.device) if halo else None
    q_ext = _thd_ext(q, zq, halo)
    k_ext = _thd_ext(k, halo_kv[:, :Hkv] if halo else None, halo)
    v_ext = _thd_ext(v, halo_kv[:, Hkv:] if halo else None, halo)
    out_ext = _thd_ext(out, zq, halo)
    dout_ext = _thd_ext(dout, zq, halo)  # no gradient flows into the halo rows
    lse_ext = lse if not halo else torch.cat(
        [torch.full((Hq, halo), float("inf"), dtype=lse.dtype, device=lse.device), lse], dim=1)
    max_len = int((cu_l[1:] - cu_l[:-1]).max())
    dq, dk, dv, dsinks = attn_bwd(q_ext, k_ext, v_ext, sinks, out_ext, dout_ext, lse_ext, window=window, rope=rope,
                                  positions=pos.to(q.device), cu_seqlens=cu_l.to(q.device), max_seqlen=max_len,
                                  softmax_scale=softmax_scale)
    dkv_halo = torch.cat([dk[:halo], dv[:halo]], dim=1) if halo else None
    return dq[halo:].contiguous(), dk[halo:].contiguous(), dv[halo:].contiguous(), dsinks, dkv_halo


def sliding_window_fwd_thd(q, k, v, sinks, cu_seqlens, window: int, rope, group=None,
                           softmax_scale: float | None = None, attn_fwd=None):
    """:func:`sliding_window_fwd` for packed inputs: this rank's ``[T_loc, H,
    D]`` tokens of a stream packed by `cu_seqlens` (global, host)."""
    rank, world = _rank_world(group)
    t_loc, _, D = q.shape
    Hkv = k.shape[1]
    halo = halo_rows(window, t_loc, world)
    got = None
    if halo:
        tail = torch.cat([k[t_loc - halo:], v[t_loc - halo:]], dim=1)
        got = _exchange(tail, (halo, 2 * Hkv, D), k.dtype, k.device, group, rank, world)
    return local_fwd_thd(q, k, v, sinks, cu_seqlens, window, rope, rank, got, softmax_scale, attn_fwd)


def sliding_window_bwd_thd(q, k, v, sinks, out, dout, lse, cu_seqlens, window: int, rope, group=None,
                           softmax_scale: float | None = None, attn_bwd=None):
    """:func:`sliding_window_bwd` for packed inputs."""
    rank, world = _rank_world(group)
    t_loc, _, D = q.shape
    Hkv = k.shape[1]
    halo = halo_rows(window, t_loc, world)
    got = None
    if halo:
        tail = torch.cat([k[t_loc - halo:], v[t_loc - halo:]], dim=1)
        got = _exchange(tail, (halo, 2 * Hkv, D), k.dtype, k.device, group, rank, world)
    dq, dk, dv, dsinks, dkv_halo = local_bwd_thd(q, k, v, sinks, out, dout, lse, cu_seqlens, window, rope, rank,
                                                 got, softmax_scale, attn_bwd)
    if halo:
        back = _exchange_back(dkv_halo, (halo, 2 * Hkv, D), dk.dtype, dk.device, group, rank, world)
        if back is not None:
            add_halo_grads(dk.unsqueeze(0), dv.unsqueeze(0), back.unsqueeze(0))
    dsinks = dsinks.clone()
    if world > 1:
        dist.all_reduce(dsinks, op=dist.ReduceOp.SUM, group=group)
    return dq, dk, dv, dsinks


def full_context_fwd(q, k, v, sinks, rope, group=None, softmax_scale: float | None = None, attn_block=None,
                     merge=None):
    """This rank's rows of the full-context attention of the whole sequence.

    q ``[B, S_loc, Hq, D]``, k / v ``[B, S_loc, Hkv, D]``: this rank's shard
    (tokens [rank S_loc, (rank + 1) S_loc) of every sequence), raw (RoPE at
    the global positions inside the block prefill).  Returns ``(out [B, S_loc,
    Hq, D], lse [B, Hq, S_loc])``.  Ring: at step s this rank holds the k / v
    block of rank (rank - s) mod R; it forwards the block to rank + 1 while it
    computes its queries against it, if that block lies at or before its shard
    (a later rank's keys are all in the future of this shard's queries).
    ``attn_block(q, k, v, q_start, k_start, rope=, softmax_scale=)`` returning
    ``(out fp32, lse)`` and ``merge(outs [n, ...], lses [n, ...], sinks)``
    returning ``(out, lse)`` default to the CUDA library."""
    attn_block = attn_block or ops.gptoss_attn_fwd_block
    merge = merge or (lambda outs, lses, snk: ops.gptoss_attn_merge(outs, lses, snk, lse=True))
    rank, world = _rank_world(group)
    s_loc = q.shape[1]
    Hkv = k.shape[2]
    held = torch.cat([k, v], dim=2).contiguous()  # the block held now: k and v heads concatenated
    outs, lses = [], []
    for step in range(world):
        src = (rank - step) % world  # whose block is held
        reqs, recv = [], None
        if step + 1 < world:  # the ring moves on while this step computes
            recv = torch.empty_like(held)
            reqs.append(dist.irecv(recv, src=_peer(group, (rank - 1) % world), group=group))
            reqs.append(dist.isend(held, dst=_peer(group, (rank + 1) % world), group=group))
        if src <= rank:
            o, l = attn_block(q, held[:, :, :Hkv], held[:, :, Hkv:], rank * s_loc, src * s_loc, rope=rope,
                              softmax_scale=softmax_scale)
            outs.append(o)
            lses.append(l)
        for r in reqs:
            r.wait()
        if recv is not None:
            held = recv  # the sent block stays referenced by `reqs` until its send completed
    return merge(torch.stack(outs), torch.stack(lses), sinks)
