"""Seeded synthetic inputs for the GPT-OSS attention core.

This module is the one thing the CUDA path and the float64 oracle share: it
draws the inputs and holds none of the method's arithmetic (no RoPE, no
softmax, no YaRN).  The shapes follow the gpt-oss-20b attention
(64 query heads, 8 key/value heads, head_dim 64; module tree on the blog page
"gpt-oss-20b 模型结构"), the sliding window of 128 tokens and the 128K
YaRN context (Transformers v4.55.0 release notes, "Architecture").  The pages
describe no workload data, so the values are N(0, 1) draws rounded to bf16
(q, k, v) or kept in fp32 (sinks).

Recipe: ``numpy.random.Generator(PCG64(seed))``; values drawn in float64 as
N(0, 1), then rounded to float32 and to bf16 (round to nearest even); draw
order [THD lengths], q, k, v, sinks.  Decode caches too large to draw on the
host in reasonable time (the two full-size decode workloads) are drawn on the
device with ``torch.Generator`` seeded the same way; the oracle then reads
the sampled sequences back from the device.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GPTOSS_ROPE = dict(base=150000.0, factor=32.0, initial_context=4096, ntk_alpha=1.0, ntk_beta=32.0)
PLAIN_ROPE = dict(base=150000.0, factor=1.0, initial_context=4096, ntk_alpha=1.0, ntk_beta=32.0)


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    window: int
    rope: dict
    seed: int
    thd_total: int = 0          # > 0: packed THD with this many tokens
    thd_len_range: tuple = (256, 8192)

    @property
    def softmax_scale(self) -> float:
        return self.D ** -0.5


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    D: int
    window: int
    rope: dict
    seed: int


# The five workloads: tiny correctness; GPT-OSS-20b-shaped sliding and full
# prefill layers; a packed THD pair (full + window 128); decode.
TINY = PrefillConfig("tiny_b1_s128_h8_kv1", 1, 128, 8, 1, 64, 0, PLAIN_ROPE, seed=0)
SLIDING = PrefillConfig("sliding_b4_s4096_w128", 4, 4096, 64, 8, 64, 128, GPTOSS_ROPE, seed=1)
FULL = PrefillConfig("full_b2_s8192", 2, 8192, 64, 8, 64, 0, GPTOSS_ROPE, seed=2)
THD_FULL = PrefillConfig("thd_t32768_full", 0, 8192, 64, 8, 64, 0, GPTOSS_ROPE, seed=3, thd_total=32768)
THD_WINDOW = PrefillConfig("thd_t32768_w128", 0, 8192, 64, 8, 64, 128, GPTOSS_ROPE, seed=3, thd_total=32768)
DECODE_B64 = DecodeConfig("decode_b64_l32768_full", 64, 32768, 64, 8, 64, 0, GPTOSS_ROPE, seed=4)
DECODE_B64_W = DecodeConfig("decode_b64_l32768_w128", 64, 32768, 64, 8, 64, 128, GPTOSS_ROPE, seed=4)
DECODE_B8 = DecodeConfig("decode_b8_l131072_full", 8, 131072, 64, 8, 64, 0, GPTOSS_ROPE, seed=5)
DECODE_B8_W = DecodeConfig("decode_b8_l131072_w128", 8, 131072, 64, 8, 64, 128, GPTOSS_ROPE, seed=5)

PREFILL_CONFIGS = [TINY, SLIDING, FULL, THD_FULL, THD_WINDOW]
DECODE_CONFIGS = [DECODE_B64, DECODE_B64_W, DECODE_B8, DECODE_B8_W]
# Variants beyond GPT-OSS's own shapes: head size 128 (32 / 8 heads, full
# rotary), and the q / k / v projection of the sliding layer's tokens.
FULL_D128 = PrefillConfig("full_d128_b2_s8192_hq32", 2, 8192, 32, 8, 128, 0, GPTOSS_ROPE, seed=6)
PROJ_HIDDEN = 2880  # GPT-OSS hidden size: q_proj 2880 -> 4096, k_proj / v_proj 2880 -> 512


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (via float32, round to nearest even); return uint16 bits."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 array holding the bf16-rounded values of ``x``."""
    return bits_to_f32(bf16_bits(x))


def thd_lengths(rng: np.random.Generator, total: int, lo: int, hi: int) -> np.ndarray:
    """Sequence lengths ~ U{lo..hi} drawn until they cover ``total`` tokens;
    the last one is cut to the remainder (it may fall below ``lo``)."""
    lens = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return np.asarray(lens, dtype=np.int64)


@dataclass
class PrefillInputs:
    q: np.ndarray          # float32 bf16-valued, [B,S,Hq,D] or [T,Hq,D]
    k: np.ndarray
    v: np.ndarray
    sinks: np.ndarray      # float32 [Hq]
    cu_seqlens: np.ndarray | None = None   # int32 [nseq+1] for THD
    extra: dict = field(default_factory=dict)


def make_prefill(cfg: PrefillConfig, seed: int | None = None, B: int | None = None,
                 S: int | None = None, thd_lengths_override=None) -> PrefillInputs:
    """Draw q, k, v, sinks for ``cfg`` (optionally with a smaller B / S)."""
    rng = np.random.Generator(np.random.PCG64(cfg.seed if seed is None else seed))
    cu = None
    if cfg.thd_total > 0 or thd_lengths_override is not None:
        if thd_lengths_override is not None:
            lens = np.asarray(thd_lengths_override, np.int64)
        else:
            lens = thd_lengths(rng, cfg.thd_total, *cfg.thd_len_range)
        cu = np.zeros(len(lens) + 1, np.int32)
        cu[1:] = np.cumsum(lens)
        T = int(cu[-1])
        lead = (T,)
    else:
        lead = (cfg.B if B is None else B, cfg.S if S is None else S)
    q = bf16_round(rng.standard_normal(lead + (cfg.Hq, cfg.D)))
    k = bf16_round(rng.standard_normal(lead + (cfg.Hkv, cfg.D)))
    v = bf16_round(rng.standard_normal(lead + (cfg.Hkv, cfg.D)))
    sinks = rng.standard_normal(cfg.Hq).astype(np.float32)
    return PrefillInputs(q, k, v, sinks, cu)


@dataclass
class DecodeInputs:
    q: np.ndarray            # float32 bf16-valued [B, Hq, D]
    k_cache: np.ndarray      # float32 bf16-valued [B, L, Hkv, D]
    v_cache: np.ndarray
    sinks: np.ndarray        # float32 [Hq]
    seqlens: np.ndarray      # int32 [B]


def make_decode_host(cfg: DecodeConfig, B: int | None = None, L: int | None = None,
                     seqlens=None, seed: int | None = None) -> DecodeInputs:
    """Host-drawn decode inputs (small shapes): caches, sinks, then q."""
    B = cfg.B if B is None else B
    L = cfg.L if L is None else L
    rng = np.random.Generator(np.random.PCG64(cfg.seed if seed is None else seed))
    kc = bf16_round(rng.standard_normal((B, L, cfg.Hkv, cfg.D)))
    vc = bf16_round(rng.standard_normal((B, L, cfg.Hkv, cfg.D)))
    sinks = rng.standard_normal(cfg.Hq).astype(np.float32)
    q = bf16_round(rng.standard_normal((B, cfg.Hq, cfg.D)))
    if seqlens is None:
        seqlens = np.full(B, L, np.int32)
    return DecodeInputs(q, kc, vc, sinks, np.asarray(seqlens, np.int32))


def make_decode_device(cfg: DecodeConfig, device, seqlens=None):
    """Device-drawn decode inputs for the full-size caches (torch Philox,
    seeded with ``cfg.seed``).  Returns torch tensors
    ``(q, k_cache, v_cache, sinks, seqlens)``: bf16, bf16, bf16, fp32, int32."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    shape = (cfg.B, cfg.L, cfg.Hkv, cfg.D)
    kc = torch.empty(shape, dtype=torch.bfloat16, device=device)
    vc = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # draw in slabs so the float32 staging stays small
    for dst in (kc, vc):
        for b in range(cfg.B):
            dst[b].copy_(torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32))
    sinks = torch.randn(cfg.Hq, generator=g, device=device, dtype=torch.float32)
    q = torch.randn((cfg.B, cfg.Hq, cfg.D), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    if seqlens is None:
        seqlens = torch.full((cfg.B,), cfg.L, dtype=torch.int32, device=device)
    else:
        seqlens = torch.as_tensor(seqlens, dtype=torch.int32, device=device)
    return q, kc, vc, sinks, seqlens


def to_torch_bf16(x: np.ndarray, device="cpu"):
    """Upload a bf16-valued float32 array as a torch bf16 tensor (exact)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(device=device).to(torch.bfloat16)
