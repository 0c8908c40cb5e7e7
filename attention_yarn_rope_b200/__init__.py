"""GPT-OSS attention core for NVIDIA B200: YaRN RoPE + grouped-query causal
softmax attention with per-head sinks, full or sliding window, prefill (BSHD,
packed THD) and split-KV decode, as hand-written sm_100a CUDA kernels behind a
C ABI (``include/gptoss.h``, ``libgptoss_attn.so``).

``attention_yarn_rope_b200.ops`` is the Python binding (torch tensors in,
kernels run on the current CUDA stream).  ``attention_yarn_rope_b200.workloads``
draws the seeded synthetic inputs.  The library is loaded on first use and
its absence is an error: nothing here computes on the CPU.
"""

__all__ = ["ops", "workloads", "build_lib"]
