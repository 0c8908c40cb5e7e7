"""Plain, slow, float64 CPU oracle for the GPT-OSS attention core.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` call it.  It shares no code, table
or constant generator with the CUDA library under
``attention_yarn_rope_b200/csrc`` and imports nothing from it.

Contents
--------
``yarn``       YaRN inverse frequencies and attention concentration
               (NeMo AutoModel ``gpt_oss.rope_utils`` page,
               ``RotaryEmbedding._compute_concentration_and_inv_freq``, which
               defers to the YaRN paper, arXiv 2309.00071).
``rope``       Half-split rotary embedding of q and k with the concentration
               applied (``gpt_oss.rope_utils`` page, ``apply_rotary_emb`` and
               ``apply_rotary_emb_qk``).
``attention``  Grouped-query causal softmax attention with a learned per-head
               sink in the denominator, full or sliding window, for BSHD,
               packed THD and single-token decode (``gpt_oss.layers`` page,
               ``GptOssAttention`` attributes ``sinks``, ``sliding_window``,
               ``softmax_scale``; Transformers v4.55.0 release notes,
               "Architecture").
``paged``      Decode over a paged KV cache (block table over a pool of
               fixed-size blocks) and appending a new token to it, reduced to
               ``attention.attn_decode`` and ``rope.rope`` (the pages describe
               generation with a cache but no cache layout).
``backward``   Gradients of the sink attention with RoPE (dq, dk, dv and the
               sink gradient): the exact derivative of ``attention``'s
               definition by the chain rule, and the RoPE adjoint
               ``rope_transpose``.  The pages define the forward and describe
               training with it; they print no backward formula.
``cp``         Attention of a query block over one key block at global
               offsets (no sink) and the log-sum-exp merge of such blocks
               with the sink folded once: the pieces of context parallelism
               for full-context layers (``cp_size`` / ``cp_rank`` on the
               ``gpt_oss.rope_utils`` page; the merge follows from the
               definition in ``attention``).
``brute``      A second, independent formulation in scalar Python loops for
               tiny shapes (complex-multiply RoPE, softmax over the logits
               with the sink appended as one more column).

Every function computes the plain definition in float64; there is no tiling,
no online softmax and no reordering beyond what a library matmul does.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, invariants, a library routine
(``torch.nn.functional.scaled_dot_product_attention`` in float64) and the
brute-force formulation; ``backward`` against central finite differences
of the forward oracle and float64 ``torch.autograd`` of a separately written
forward.  The one reading the pages leave open and no
invariant can decide -- the shape of the YaRN ramp between the two correction
dimensions -- is selectable (``ramp="index"`` is the adopted reading,
``ramp="paper"`` the YaRN paper's gamma(r)); the choice between them is
parity unpinned by the pages.
"""
