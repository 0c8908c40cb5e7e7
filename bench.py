#!/usr/bin/env python
"""Benchmark of the GPT-OSS attention core on B200.

Default workload (one "step"): the GPT-OSS-20b-shaped sliding-window layer
prefill -- B=4, S=4096, 64 query / 8 kv heads, head_dim 64, window 128,
YaRN RoPE (base 150000, factor 32, L0 4096, alpha 1, beta 32) fused into the
attention kernel, per-head sinks -- one ``gptoss_attn_fwd`` launch.

Prints ONE JSON line: ``value`` is whole-job sink-attention TFLOP/s (4*D
FLOP per visible (query, key) pair per head, summed over all ranks),
``e2e`` the same metric through the public API with pinned host buffers and
the host<->device copies inside the timed region, ``roofline`` the dominant
kernel against the measured HBM peak, ``cpu_baseline`` the float64 oracle on
a bounded sample, and ``per_config`` the other workloads (full prefill, THD
pair, decode) measured the same way.

``--impl reference`` times the float64 CPU oracle on the same workload
(bounded sample per step) and prints the same line with ``"impl":
"reference"``.

Multi-GPU (``torchrun --nproc-per-node N bench.py --gpus N``): one process per
GPU, each running its own replica of the workload (the path has no exchange
step, so there is no collective in the data path); the time is the max over
ranks and ``value`` sums the work of all ranks (weak scaling).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sink-attn fwd TFLOP/s (prefill) & HBM GB/s (decode), % of B200 roofline"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def visible_pairs(lens, window):
    """Number of visible (query, key) pairs of causal attention over sequences
    of the given lengths (window 0 = full)."""
    tot = 0
    for n in lens:
        n = int(n)
        if window <= 0 or window >= n:
            tot += n * (n + 1) // 2
        else:
            tot += window * (window + 1) // 2 + (n - window) * window
    return tot


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def mark(self):
        return time.time()

    def stop(self, t_lo=None, t_hi=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[5:]))
                except Exception:
                    continue
        os.unlink(self.tmp.name)
        window = "timed"
        sel = [r for r in rows if t_lo is not None and t_lo - 1 <= r[0] <= t_hi + 1]
        if not sel:
            sel, window = rows, "warmup+timed"
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        mhz = sorted(r[1] for r in sel)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in sel:
            flags = r[3][1:]
            for n, f in zip(names, flags):
                if f.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": max(r[2] for r in sel), "reasons": sorted(reasons),
                "samples": len(sel), "window": window}


# ----------------------------------------------------------------------------
# timing helpers
# ----------------------------------------------------------------------------
def aggregate_ranks(torch, dist, device, ms_local, work_local):
    """Whole-job view of one timed region: the time is the max over ranks
    (every rank waited at a barrier before and after it), the work the sum.
    Single process: returned unchanged."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms_local), float(work_local)
    dist.barrier()
    t = torch.tensor([float(ms_local)], dtype=torch.float64, device=device)
    w = torch.tensor([float(work_local)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t.item()), float(w.item())


def timed_steps(torch, fn, steps, stream, flush=None):
    """Device time (ms) of `steps` calls of fn on `stream`, CUDA events on that
    stream; with `flush`, L2 is overwritten between calls (outside the timing)."""
    if flush is None:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(steps):
            fn()
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end)
    total = 0.0
    for _ in range(steps):
        flush()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        fn()
        end.record(stream)
        end.synchronize()
        total += start.elapsed_time(end)
    return total


# ----------------------------------------------------------------------------
# workloads (our arm)
# ----------------------------------------------------------------------------
def prefill_case(torch, ops, cfg, device, seed_offset=0):
    """Device inputs and a step closure for one prefill workload."""
    from attention_yarn_rope_b200.workloads import make_prefill, to_torch_bf16

    x = make_prefill(cfg, seed=cfg.seed + seed_offset)
    q, k, v = (to_torch_bf16(a, device) for a in (x.q, x.k, x.v))
    sinks = torch.from_numpy(x.sinks).to(device)
    rope = ops.RopeConfig.from_dict(cfg.rope, rotary_dim=cfg.D)
    out = torch.empty_like(q)
    # k is rotated once per call into this workspace (allocated once, outside the timing)
    ws = torch.empty(ops.gptoss_attn_fwd_workspace_size(x.k.shape[0] * x.k.shape[1] if x.k.ndim == 4 else x.k.shape[0],
                                                        cfg.Hkv, cfg.D), dtype=torch.uint8, device=device)
    if x.cu_seqlens is not None:
        lens = [int(a) for a in (x.cu_seqlens[1:] - x.cu_seqlens[:-1])]
        cu = torch.from_numpy(x.cu_seqlens).to(device)
        max_len = max(lens)

        def step():
            ops.gptoss_attn_fwd(q, k, v, sinks, window=cfg.window, rope=rope, cu_seqlens=cu, max_seqlen=max_len,
                                out=out, workspace=ws)
    else:
        lens = [cfg.S] * cfg.B
        cu = None

        def step():
            ops.gptoss_attn_fwd(q, k, v, sinks, window=cfg.window, rope=rope, out=out, workspace=ws)
    pairs = visible_pairs(lens, cfg.window) * cfg.Hq
    flops = 4 * cfg.D * pairs
    io_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, out))
    return dict(x=x, q=q, k=k, v=v, sinks=sinks, out=out, cu=cu, step=step, flops=flops, bytes=io_bytes,
                pairs=pairs, rope=rope, lens=lens, ws=ws)


def proj_case(torch, ops, device, B=4, S=4096, Hq=64, Hkv=8, D=64, seed=7):
    """gptoss_qkv_rope over B x S tokens of GPT-OSS's hidden size: Linear-like
    weights (N(0, 1 / hidden)), biases N(0, 0.01), x N(0, 1), all bf16."""
    from attention_yarn_rope_b200.workloads import GPTOSS_ROPE, PROJ_HIDDEN

    gen = torch.Generator(device=device).manual_seed(seed)
    N = (Hq + 2 * Hkv) * D
    x = torch.randn((B, S, PROJ_HIDDEN), generator=gen, device=device).to(torch.bfloat16)
    w = (torch.randn((N, PROJ_HIDDEN), generator=gen, device=device) / PROJ_HIDDEN ** 0.5).to(torch.bfloat16)
    b = (torch.randn((N,), generator=gen, device=device) * 0.1).to(torch.bfloat16)
    rope = ops.RopeConfig.from_dict(GPTOSS_ROPE, rotary_dim=D)
    q = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=device)
    k = torch.empty((B, S, Hkv, D), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    ws = torch.empty(ops.gptoss_qkv_rope_workspace_size(B * S, D), dtype=torch.uint8, device=device)

    def step():
        ops.gptoss_qkv_rope(x, w, b, Hq, Hkv, rope=rope, q_out=q, k_out=k, v_out=v, workspace=ws)
    return dict(step=step, flops=2 * B * S * PROJ_HIDDEN * N)


def bwd_case(torch, ops, cfg, device):
    """The backward of one prefill workload: the forward runs once outside the
    step for out / lse; the step is one gptoss_attn_bwd call (dq, dk, dv,
    dsinks) with a preallocated workspace.  FLOP = 2.5 x the forward's (5
    products of 2 D per visible pair and head)."""
    case = prefill_case(torch, ops, cfg, device)
    q, k, v, sinks, rope = case["q"], case["k"], case["v"], case["sinks"], case["rope"]
    kw = {} if case["cu"] is None else dict(cu_seqlens=case["cu"], max_seqlen=max(case["lens"]))
    out, lse = ops.gptoss_attn_fwd(q, k, v, sinks, window=cfg.window, rope=rope, return_lse=True, **kw)
    gen = torch.Generator(device=device).manual_seed(cfg.seed + 100)
    dout = torch.randn(q.shape, generator=gen, device=device).to(torch.bfloat16)
    total = q.shape[0] * q.shape[1] if q.dim() == 4 else q.shape[0]
    ws = torch.empty(ops.gptoss_attn_bwd_workspace_size(total, cfg.Hq, cfg.Hkv, cfg.D), dtype=torch.uint8,
                     device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsinks = torch.empty(cfg.Hq, dtype=torch.float32, device=device)

    def step():
        ops.gptoss_attn_bwd(q, k, v, sinks, out, dout, lse, window=cfg.window, rope=rope, dq=dq, dk=dk, dv=dv,
                            dsinks=dsinks, workspace=ws, **kw)
    io = sum(t.numel() * t.element_size() for t in (q, k, v, out, dout, dq, dk, dv))
    return dict(step=step, flops=2.5 * case["flops"], bytes=io)


def decode_case(torch, ops, cfg, device):
    from attention_yarn_rope_b200.workloads import make_decode_device

    q, kc, vc, sinks, seqlens = make_decode_device(cfg, device)
    rope = ops.RopeConfig.from_dict(cfg.rope)
    out = torch.empty_like(q)
    ws = torch.empty(ops.gptoss_attn_decode_workspace_size(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.D),
                     dtype=torch.uint8, device=device)

    def step():
        ops.gptoss_attn_decode(q, kc, vc, seqlens, sinks, window=cfg.window, rope=rope, out=out, workspace=ws)
    span = cfg.L if cfg.window == 0 else min(cfg.window, cfg.L)
    kv_bytes = 2 * cfg.B * span * cfg.Hkv * cfg.D * 2
    io_bytes = kv_bytes + 2 * q.numel() * 2
    return dict(step=step, bytes=io_bytes, kv_bytes=kv_bytes, flops=4 * cfg.D * cfg.B * cfg.Hq * span,
                q=q, kc=kc, vc=vc, sinks=sinks, rope=rope, out=out, ws=ws)


def decode_graph_us(torch, ops, cfg, case, flush, calls=100, reps=5):
    """Per-call time of `calls` back-to-back windowed decode calls replayed from
    one CUDA graph, each call on a disjoint window of the cache (call c sees
    the slots ending at L - window * c), L2 flushed before every replay."""
    dev = case["q"].device
    lens = [torch.full((cfg.B,), cfg.L - cfg.window * c, dtype=torch.int32, device=dev) for c in range(calls)]

    def call(c):
        ops.gptoss_attn_decode(case["q"], case["kc"], case["vc"], lens[c], case["sinks"], window=cfg.window,
                               rope=case["rope"], out=case["out"], workspace=case["ws"])

    for c in range(calls):  # warm every path once outside the capture
        call(c)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in range(calls):
            call(c)
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(reps):
        flush()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        g.replay()
        end.record(stream)
        end.synchronize()
        times.append(start.elapsed_time(end) * 1e3 / calls)
    del g
    return sorted(times)[len(times) // 2]


def run_ours(args, torch, dist, rank, world, device):
    from attention_yarn_rope_b200 import ops
    from attention_yarn_rope_b200.workloads import (
        DECODE_B8, DECODE_B8_W, DECODE_B64, DECODE_B64_W, FULL, FULL_D128, SLIDING, THD_FULL, THD_WINDOW)

    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    cfg = SLIDING
    case = prefill_case(torch, ops, cfg, device, seed_offset=rank)
    for _ in range(args.warmup):
        case["step"]()
    torch.cuda.synchronize()
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(torch.cuda.current_device())).split(",")[0]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else torch.cuda.current_device()
    clk = ClockSampler(gpu_index if world == 1 else torch.cuda.current_device())
    clk.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_lo = time.time()
    ms = timed_steps(torch, case["step"], args.steps, stream)
    torch.cuda.synchronize()
    t_hi = time.time()
    ms, job_flops = aggregate_ranks(torch, dist, device, ms, case["flops"] * args.steps)
    clocks = clk.stop(t_lo, t_hi)
    per_step_ms = ms / args.steps
    value = job_flops / (ms * 1e-3) / 1e12

    # ---- end to end through the public API, host buffers, copies inside ----
    # Every step uploads its inputs from pinned host memory and reads its
    # output back.  Two device buffer sets and two copy streams pipeline the
    # steps: step n+1's upload and step n-1's download run on the copy engines
    # while step n's kernels run.
    h_q = case["q"].cpu().pin_memory()
    h_k = case["k"].cpu().pin_memory()
    h_v = case["v"].cpu().pin_memory()
    h_s = case["sinks"].cpu().pin_memory()
    h_os = [torch.empty(case["out"].shape, dtype=case["out"].dtype).pin_memory() for _ in range(2)]
    sets = [tuple(torch.empty_like(t) for t in (case["q"], case["k"], case["v"], case["sinks"], case["out"]))
            for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(nsteps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        h2d_s.wait_event(start)
        d2h_s.wait_event(start)
        for n in range(nsteps):
            b = n % 2
            d_q, d_k, d_v, d_s, d_o = sets[b]
            with torch.cuda.stream(h2d_s):
                if n >= 2:
                    h2d_s.wait_event(comp_done[b])  # step n-2 has read this set's inputs
                d_q.copy_(h_q, non_blocking=True)
                d_k.copy_(h_k, non_blocking=True)
                d_v.copy_(h_v, non_blocking=True)
                d_s.copy_(h_s, non_blocking=True)
                in_ready[b].record(h2d_s)
            stream.wait_event(in_ready[b])
            if n >= 2:
                stream.wait_event(d2h_done[b])  # step n-2's output has left this set
            ops.gptoss_attn_fwd(d_q, d_k, d_v, d_s, window=cfg.window, rope=case["rope"], out=d_o,
                                workspace=case["ws"], stream=stream)
            comp_done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[b])
                h_os[b].copy_(d_o, non_blocking=True)
                d2h_done[b].record(d2h_s)
        for b in range(2):
            stream.wait_event(d2h_done[b])
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end)

    e2e_run(3)
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 50))
    if world > 1:
        dist.barrier()
    ems = e2e_run(e2e_steps)
    ems, e2e_flops = aggregate_ranks(torch, dist, device, ems, case["flops"] * e2e_steps)
    e2e_value = e2e_flops / (ems * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_s))
    d2h = h_os[0].numel() * h_os[0].element_size()

    achieved_gbs = case["bytes"] / (per_step_ms * 1e-3) / 1e9
    # DRAM bytes of the step's two kernels (one ncu capture each, taken on
    # their current sources), summed like the duration they are set against
    by_kernel = {k: read_traffic(k, cfg.name) for k in ("rope_qk_kernel<true>", "attn_fwd_kernel")}
    traffic = None if None in by_kernel.values() else sum(by_kernel.values())
    roofline = {"kernel": "attn_fwd_kernel", "bound": "hbm", "achieved": round(achieved_gbs, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
                "peak_source": peaks["source"], "traffic": traffic, "traffic_by_kernel": by_kernel,
                "algorithmic_bytes_per_launch": case["bytes"],
                "duration": "whole step: k rotation into the workspace + attention kernel",
                "tflops": round(case["flops"] / (per_step_ms * 1e-3) / 1e12, 2)}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "S": cfg.S, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D,
                   "window": cfg.window,
                   "rope": "yarn base 150000 factor 32 L0 4096 alpha 1 beta 32 (k once into a workspace, q in-kernel)",
                   "global_batch": cfg.B * world, "seq_len": cfg.S, "parallelism": f"replicas{world}",
                   "l2": f"inputs {case['bytes'] / 1e6:.0f} MB > L2 126 MB, no flush"},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": round(ems / e2e_steps, 4),
                "pipeline": "2 buffer sets: step n+1 upload and step n-1 download overlap step n"},
        "gpu_launches": 2 * args.steps,  # rope_qk_kernel<true> (k into the workspace) + attn_fwd_kernel
        "clocks": clocks,
        "roofline": roofline,
    }
    del h_q, h_k, h_v, h_os, sets, case
    torch.cuda.empty_cache()

    if world == 1 and not args.no_extras:
        line["per_config"] = per_config(torch, ops, device, stream, peaks,
                                        [FULL, THD_FULL, THD_WINDOW, FULL_D128],
                                        [DECODE_B64, DECODE_B64_W, DECODE_B8, DECODE_B8_W], args,
                                        bwd_cfgs=[SLIDING, FULL])
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(SLIDING, budget_s=args.cpu_seconds)
    return line


def per_config(torch, ops, device, stream, peaks, prefill_cfgs, decode_cfgs, args, bwd_cfgs=()):
    # the denominators of every frac_of_* below: MEASURED_PEAKS.json when the
    # file is present ("measured"), else the pool's earlier figures ("fallback")
    res = {"peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"], "source": peaks["source"]}}
    reps = max(3, min(args.steps, 20))
    for cfg in prefill_cfgs:
        case = prefill_case(torch, ops, cfg, device)
        for _ in range(3):
            case["step"]()
        torch.cuda.synchronize()
        ms = timed_steps(torch, case["step"], reps, stream) / reps
        tf = case["flops"] / (ms * 1e-3) / 1e12
        gbs = case["bytes"] / (ms * 1e-3) / 1e9
        res[cfg.name] = {"ms": round(ms, 4), "tflops": round(tf, 2), "frac_of_bf16_peak": round(
            tf / peaks["bf16_tflops"], 4), "frac_of_2250_spec": round(tf / 2250.0, 4), "gbs": round(gbs, 1),
            "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4), "visible_pairs": case["pairs"],
            "flops": case["flops"], "bytes": case["bytes"], "launches_per_call": 2}
        del case
        torch.cuda.empty_cache()
    # the q / k / v projections with RoPE in the GEMM epilogue, for the
    # sliding layer's 16384 tokens (x [4, 4096, 2880], GPT-OSS's 64 / 8 heads)
    pj = proj_case(torch, ops, device)
    for _ in range(3):
        pj["step"]()
    torch.cuda.synchronize()
    ms = timed_steps(torch, pj["step"], reps, stream) / reps
    tf = pj["flops"] / (ms * 1e-3) / 1e12
    res["qkv_rope_b4_s4096_h2880"] = {"ms": round(ms, 4), "tflops": round(tf, 2),
                                     "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4), "flops": pj["flops"],
                                     "launches_per_call": 2, "note": "x W^T + b on tcgen05, RoPE of q and k in the epilogue"}
    del pj
    torch.cuda.empty_cache()
    # backward (training): dq, dk, dv, dsinks of the forward's output; 5
    # products per visible pair and head (S and dP recomputed, dV, dK, dQ)
    for cfg in bwd_cfgs:
        case = bwd_case(torch, ops, cfg, device)
        for _ in range(3):
            case["step"]()
        torch.cuda.synchronize()
        ms = timed_steps(torch, case["step"], reps, stream) / reps
        tf = case["flops"] / (ms * 1e-3) / 1e12
        res["bwd_" + cfg.name] = {"ms": round(ms, 4), "tflops": round(tf, 2),
                                  "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
                                  "gbs_io": round(case["bytes"] / (ms * 1e-3) / 1e9, 1), "flops": case["flops"],
                                  "io_bytes": case["bytes"], "launches_per_call": "4 (5 with split sweeps)",
                                  "note": "dK / dV on tcgen05 (TMEM); dQ on tcgen05 for long sweeps, mma.sync for short ones"}
        del case
        torch.cuda.empty_cache()
    flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    for cfg in decode_cfgs:
        case = decode_case(torch, ops, cfg, device)
        for _ in range(3):
            case["step"]()
        torch.cuda.synchronize()
        small = case["kv_bytes"] < 4 * L2_BYTES
        ms = timed_steps(torch, case["step"], reps, stream,
                         flush=(lambda: flush_buf.fill_(1)) if small else None) / reps
        gbs = case["bytes"] / (ms * 1e-3) / 1e9
        res[cfg.name] = {"ms": round(ms, 4), "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
                         "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4), "kv_bytes": case["kv_bytes"],
                         "l2": "flushed between calls" if small else "cache > L2",
                         "launches_per_call": 1 if cfg.window and cfg.window <= 256 else 2}
        if cfg.window and cfg.window * 100 < cfg.L:
            try:
                gus = decode_graph_us(torch, ops, cfg, case, lambda: flush_buf.fill_(1))
                res[cfg.name]["graph_us_per_call"] = round(gus, 2)
                res[cfg.name]["graph_gbs"] = round(case["bytes"] / (gus * 1e-6) / 1e9, 1)
                res[cfg.name]["graph"] = "100 calls on disjoint windows in one CUDA graph, L2 flushed per replay"
            except Exception as e:  # report the measurement as missing, not the run as failed
                res[cfg.name]["graph_us_per_call"] = None
                res[cfg.name]["graph_error"] = str(e)[:200]
        del case
        torch.cuda.empty_cache()
    # paged decode: the B=64 x 32768 cache seen as 256-token blocks behind a
    # random block table (same bytes, read through the page indirection)
    for cfg in decode_cfgs[:1]:
        case = decode_case(torch, ops, cfg, device)
        bs = 256
        nblk = cfg.B * cfg.L // bs
        gen = torch.Generator(device="cpu").manual_seed(7)
        table = torch.randperm(nblk, generator=gen).reshape(cfg.B, cfg.L // bs).to(torch.int32).to(device)
        kp = case["kc"].view(nblk, bs, cfg.Hkv, cfg.D)
        vp = case["vc"].view(nblk, bs, cfg.Hkv, cfg.D)
        lens = torch.full((cfg.B,), cfg.L, dtype=torch.int32, device=device)

        def pstep():
            ops.gptoss_attn_decode_paged(case["q"], kp, vp, table, lens, case["sinks"], window=cfg.window,
                                         rope=case["rope"], out=case["out"], workspace=case["ws"])
        for _ in range(3):
            pstep()
        torch.cuda.synchronize()
        ms = timed_steps(torch, pstep, reps, stream) / reps
        gbs = case["bytes"] / (ms * 1e-3) / 1e9
        res[f"decode_paged_b{cfg.B}_l{cfg.L}_bs{bs}_full"] = {
            "ms": round(ms, 4), "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
            "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4), "kv_bytes": case["kv_bytes"],
            "block_size": bs, "table": f"random permutation of the {nblk} blocks", "launches_per_call": 2}
        # four new tokens per sequence (draft tokens checked in one call): the
        # four share each CTA's pass over the cache (32 query rows per kv head)
        q_len = 4
        q4 = case["q"][:, None].repeat(1, q_len, 1, 1).contiguous()  # the seeded queries, one per new token
        o4 = torch.empty_like(q4)
        ws4 = torch.empty(ops.gptoss_attn_decode_workspace_size(cfg.B * q_len, cfg.L, cfg.Hq, cfg.Hkv, cfg.D),
                          dtype=torch.uint8, device=device)

        def mstep():
            ops.gptoss_attn_decode_paged(q4, kp, vp, table, lens, case["sinks"], window=cfg.window,
                                         rope=case["rope"], out=o4, workspace=ws4)
        for _ in range(3):
            mstep()
        torch.cuda.synchronize()
        ms4 = timed_steps(torch, mstep, reps, stream) / reps
        res[f"decode_paged_b{cfg.B}_l{cfg.L}_bs{bs}_qlen{q_len}_full"] = {
            "ms": round(ms4, 4), "us": round(ms4 * 1e3, 2), "q_len": q_len,
            "cache_read_once_gbs": round(case["bytes"] / (ms4 * 1e-3) / 1e9, 1),
            "x_single_token_time": round(ms4 / ms, 3), "launches_per_call": 2}
        del case, kp, vp, q4, o4, ws4
        torch.cuda.empty_cache()
    return res


def read_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel's sources as they are now (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = f"{kernel} {workload} "
    src_hash = kernel_src_hash(kernel)
    with open(path) as fh:
        for line in fh:
            if line.startswith(want):
                parts = line.split()
                if len(parts) >= 4 and parts[3] == src_hash:
                    return int(parts[2])
    return None


# The sources each measured kernel is built from: the include closure of the
# header that defines it, plus the host file that launches it (its own text
# only: the library source also includes the other kernels' headers).
_KERNEL_SOURCES = {
    "attn_fwd_kernel": ("fwd_pipeline.cuh", "fwd_host.cuh"),
    "rope_qk_kernel<true>": ("rope_qk.cuh", "fwd_host.cuh"),
    "attn_decode_split_kernel": ("attn_decode.cuh", "decode_host.cuh"),
    "attn_bwd_dkdv_tc_kernel": ("attn_bwd_tc.cuh", "bwd_host.cuh"),
    "attn_fwd128_kernel": ("fwd128.cuh", "fwd_host.cuh"),
    "qkv_rope_kernel": ("qkv_rope.cuh", "qkv_rope.cuh"),  # launched from its own header
}


def _code_only(text: str) -> str:
    """C / C++ source without its comments (string literals kept): the hash
    follows the code, not its documentation."""
    import re

    pat = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    return pat.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)


def kernel_src_hash(kernel):
    import hashlib
    import re

    csrc = os.path.join(ROOT, "attention_yarn_rope_b200", "csrc")
    inc = os.path.join(ROOT, "include")
    root, launcher = _KERNEL_SOURCES[kernel]

    def path_of(f):
        return os.path.join(csrc, f) if os.path.exists(os.path.join(csrc, f)) else os.path.join(inc, f)

    seen, todo = [], [root]
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.append(f)
        with open(path_of(f)) as fh:
            todo += re.findall(r'^#include "([^"]+)"', fh.read(), flags=re.M)
    h = hashlib.sha256()
    for f in sorted(seen) + [launcher]:
        with open(path_of(f)) as fh:
            code = " ".join(_code_only(fh.read()).split())  # whitespace-insensitive too
        h.update(f.encode() + b"\0" + code.encode())
    return h.hexdigest()[:12]


# ----------------------------------------------------------------------------
# the float64 oracle on the host cores (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
def _oracle_unit(x, cfg, b, g, tables):
    """Oracle prefill of one (batch row, kv group): G query heads, all rows.
    Returns the visible pairs it covered."""
    import numpy as np

    from oracle.attention import sink_attention_sequence
    from oracle.rope import rope

    G = cfg.Hq // cfg.Hkv
    pos = np.arange(cfg.S)
    qr = rope(x.q[b][:, g * G:(g + 1) * G], pos, *tables)
    kr = rope(x.k[b][:, g:g + 1], pos, *tables)
    sink_attention_sequence(qr, kr, x.v[b][:, g:g + 1], x.sinks[g * G:(g + 1) * G], cfg.softmax_scale, cfg.window)
    return visible_pairs([cfg.S], cfg.window) * G


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _tables_of(cfg):
    from oracle.yarn import yarn_inv_freq_and_concentration

    r = cfg.rope
    return yarn_inv_freq_and_concentration(cfg.D, r["base"], r["factor"], r["initial_context"], r["ntk_alpha"],
                                           r["ntk_beta"])


def _oracle_prefill_whole(cfg):
    """The oracle's whole output for a prefill workload: seconds, visible pairs."""
    import numpy as np

    from attention_yarn_rope_b200.workloads import make_prefill
    from oracle.attention import attn_fwd_bshd, attn_fwd_thd

    x = make_prefill(cfg)
    tables = _tables_of(cfg)
    t0 = time.perf_counter()
    if x.cu_seqlens is not None:
        attn_fwd_thd(x.q, x.k, x.v, x.sinks, x.cu_seqlens, cfg.softmax_scale, cfg.window, rope_tables=tables)
        pairs = visible_pairs(np.diff(x.cu_seqlens), cfg.window) * cfg.Hq
    else:
        attn_fwd_bshd(x.q, x.k, x.v, x.sinks, cfg.softmax_scale, cfg.window, rope_tables=tables)
        pairs = visible_pairs([cfg.S] * cfg.B, cfg.window) * cfg.Hq
    return time.perf_counter() - t0, pairs


def _oracle_prefill_sample(cfg, budget_s):
    """The oracle on (sequence, kv group) units of a prefill workload until
    about ``budget_s`` seconds; returns seconds, pairs covered, pairs of the
    whole workload and a description of the sample."""
    import numpy as np

    from attention_yarn_rope_b200.workloads import make_prefill
    from oracle.attention import sink_attention_sequence
    from oracle.rope import rope

    x = make_prefill(cfg)
    tables = _tables_of(cfg)
    G = cfg.Hq // cfg.Hkv
    if x.cu_seqlens is not None:
        cu = x.cu_seqlens
        seqs = [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
        total = visible_pairs(np.diff(cu), cfg.window) * cfg.Hq
        get = lambda s: (x.q[seqs[s][0]:seqs[s][1]], x.k[seqs[s][0]:seqs[s][1]], x.v[seqs[s][0]:seqs[s][1]])
    else:
        seqs = [(0, cfg.S)] * cfg.B
        total = visible_pairs([cfg.S] * cfg.B, cfg.window) * cfg.Hq
        get = lambda s: (x.q[s], x.k[s], x.v[s])
    # shortest sequences first for a packed stream, so the sample spans several
    order = sorted(range(len(seqs)), key=lambda s: seqs[s][1] - seqs[s][0])
    pairs, n = 0, 0
    t0 = time.perf_counter()
    for s in order:
        q, k, v = get(s)
        L = q.shape[0]
        pos = np.arange(L)
        for g in range(cfg.Hkv):
            qr = rope(q[:, g * G:(g + 1) * G], pos, *tables)
            kr = rope(k[:, g:g + 1], pos, *tables)
            sink_attention_sequence(qr, kr, v[:, g:g + 1], x.sinks[g * G:(g + 1) * G], cfg.softmax_scale,
                                    cfg.window)
            pairs += visible_pairs([L], cfg.window) * G
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return dt, pairs, total, f"{n} (sequence, kv-group) units"


def _oracle_decode_sample(cfg, n_seq):
    """The decode oracle on ``n_seq`` host-drawn sequences of the workload's
    cache length; returns seconds and the visible K + V bytes they read."""
    from attention_yarn_rope_b200.workloads import make_decode_host
    from oracle.attention import attn_decode

    x = make_decode_host(cfg, B=n_seq)
    tables = _tables_of(cfg)
    t0 = time.perf_counter()
    attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.sinks, cfg.D ** -0.5, cfg.window, rope_tables=tables)
    dt = time.perf_counter() - t0
    vis = min(cfg.L, cfg.window) if cfg.window > 0 else cfg.L
    return dt, n_seq * vis * cfg.Hkv * cfg.D * 2 * 2


def cpu_baseline(cfg, budget_s=15.0, per_config=True):
    """Times the oracle as it stands on the host cores: the whole output of
    the sliding-window workload (the headline figure), and for every other
    workload its whole output (windowed THD stream) or a bounded sample with
    the whole-workload time extrapolated from it."""
    from attention_yarn_rope_b200.workloads import (
        DECODE_B8, DECODE_B8_W, DECODE_B64, DECODE_B64_W, FULL, THD_FULL, THD_WINDOW)

    cores = _host_cores()
    dt, pairs = _oracle_prefill_whole(cfg)
    tf = 4 * cfg.D * pairs / dt / 1e12
    res = {"value": round(tf, 6), "unit": UNIT, "cores": cores, "blas_threads": _blas_threads(), "kind": "oracle",
           "sample": f"the whole output of {cfg.name} ({cfg.B} x {cfg.S} rows x {cfg.Hq} heads), float64 NumPy, "
                     f"{dt:.1f} s on {cores} host cores"}
    if not per_config:
        return res
    pc = {cfg.name: {"seconds": round(dt, 2), "tflops": round(tf, 6), "work": "whole output"}}
    dt, pairs = _oracle_prefill_whole(THD_WINDOW)
    pc[THD_WINDOW.name] = {"seconds": round(dt, 2), "tflops": round(4 * THD_WINDOW.D * pairs / dt / 1e12, 6),
                           "work": "whole output"}
    for c in (FULL, THD_FULL):
        dt, pairs, total, what = _oracle_prefill_sample(c, budget_s / 2)
        tf = 4 * c.D * pairs / dt / 1e12
        pc[c.name] = {"seconds": round(dt, 2), "tflops": round(tf, 6), "work": f"sample: {what}",
                      "est_whole_output_seconds": round(dt * total / pairs, 1)}
    for c, n in ((DECODE_B64, 2), (DECODE_B64_W, 64), (DECODE_B8, 1), (DECODE_B8_W, 8)):
        dt, nbytes = _oracle_decode_sample(c, n)
        pc[c.name] = {"seconds": round(dt, 3), "gbs": round(nbytes / dt / 1e9, 4),
                      "work": f"{n} of {c.B} sequences" + ("" if n == c.B else " (host-drawn, same shape)"),
                      "est_whole_output_seconds": round(dt * c.B / n, 2)}
    res["per_config"] = pc
    return res


def run_reference(args):
    """The reference arm: the float64 oracle on this machine's host cores,
    one (batch row, kv group) unit of the default workload per step."""
    from attention_yarn_rope_b200.workloads import SLIDING, make_prefill
    from oracle.yarn import yarn_inv_freq_and_concentration

    cfg = SLIDING
    x = make_prefill(cfg)
    r = cfg.rope
    tables = yarn_inv_freq_and_concentration(cfg.D, r["base"], r["factor"], r["initial_context"], r["ntk_alpha"],
                                             r["ntk_beta"])
    units = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    for i in range(args.warmup):
        _oracle_unit(x, cfg, *units[i % len(units)], tables)
    pairs = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        pairs += _oracle_unit(x, cfg, *units[i % len(units)], tables)
    dt = time.perf_counter() - t0
    value = 4 * cfg.D * pairs / dt / 1e12
    sample = (f"one (batch row, kv-group) unit per step: {cfg.Hq // cfg.Hkv} query heads x {cfg.S} rows of "
              f"{cfg.name}, float64 NumPy")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / max(1, args.steps) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "S": cfg.S, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D,
                   "window": cfg.window, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def profile_case(args):
    """Launch one workload's kernel(s) warmup + steps times and exit (a small,
    self-contained target for ncu captures)."""
    import dataclasses

    import torch

    from attention_yarn_rope_b200 import ops
    from attention_yarn_rope_b200 import workloads as wl

    device = "cuda:0"
    if args.profile_case == "qkv_rope_b4_s4096_h2880":  # the fused projection (a GEMM, not a PrefillConfig)
        B = args.profile_batch if args.profile_batch is not None else 4
        case = proj_case(torch, ops, device, B=B)
        for _ in range(args.warmup + args.steps):
            case["step"]()
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": args.profile_case, "B": B, "launches": args.warmup + args.steps,
                          "flops_per_launch": case["flops"]}))
        return 0
    cfgs = {c.name: c for c in wl.PREFILL_CONFIGS + wl.DECODE_CONFIGS + [wl.FULL_D128]}
    cfg = cfgs[args.profile_case]
    if args.profile_batch is not None:
        cfg = dataclasses.replace(cfg, B=args.profile_batch)
    if isinstance(cfg, wl.DecodeConfig):
        case = decode_case(torch, ops, cfg, device)
    elif args.profile_bwd:
        case = bwd_case(torch, ops, cfg, device)
    else:
        case = prefill_case(torch, ops, cfg, device)
    for _ in range(args.warmup + args.steps):
        case["step"]()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": cfg.name, "B": cfg.B, "launches": args.warmup + args.steps,
                      "bytes_per_launch": case["bytes"], "flops_per_launch": case["flops"]}))
    return 0


# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-config measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-case", default=None,
                    help="only launch this workload's kernel warmup+steps times (for ncu), e.g. "
                         "sliding_b4_s4096_w128, full_b2_s8192, decode_b64_l32768_full, "
                         "full_d128_b2_s8192_hq32, qkv_rope_b4_s4096_h2880; no timing")
    ap.add_argument("--profile-batch", type=int, default=None, help="smaller batch for --profile-case")
    ap.add_argument("--profile-bwd", action="store_true",
                    help="with --profile-case of a prefill workload: launch its backward instead")
    args = ap.parse_args()
    if args.profile_case:
        return profile_case(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch

    dist = None
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        import datetime

        import torch.distributed as dist

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(device))
    try:
        line = run_ours(args, torch, dist, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
