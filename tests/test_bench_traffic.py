"""The benchmark's DRAM-traffic figures (profiles/traffic.txt) are reported
only while the kernels they were captured on are unchanged: each line holds
the hash of its kernel's sources (the include closure of the header that
defines it plus its host launcher, comments and whitespace removed).  These CPU checks keep that
honest: the headline step's two kernels have a figure for the current
sources, and the hash moves with the code it covers and with nothing else."""

import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_headline_kernels_have_current_traffic():
    for kernel in ("attn_fwd_kernel", "rope_qk_kernel<true>"):
        assert bench.read_traffic(kernel, "sliding_b4_s4096_w128") is not None, kernel


def test_hash_covers_the_kernel_sources_only(tmp_path, monkeypatch):
    # a private copy of the tree: edit a file outside attn_fwd_kernel's
    # closure (the decode kernel) and one inside (the softmax header)
    for d in ("attention_yarn_rope_b200/csrc", "include"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_src_hash("attn_fwd_kernel")
    assert h0 == bench.kernel_src_hash("attn_fwd_kernel")
    with open(tmp_path / "attention_yarn_rope_b200/csrc/attn_decode.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_src_hash("attn_fwd_kernel") == h0
    # comments and layout are documentation: the hash ignores them
    with open(tmp_path / "attention_yarn_rope_b200/csrc/fwd_softmax.cuh", "a") as f:
        f.write("\n// a comment\n/* another */\n\n")
    assert bench.kernel_src_hash("attn_fwd_kernel") == h0
    with open(tmp_path / "include/gptoss.h", "a") as f:
        f.write("\n/* a documentation change */\n")
    assert bench.kernel_src_hash("attn_fwd_kernel") == h0
    # code is not
    with open(tmp_path / "attention_yarn_rope_b200/csrc/fwd_softmax.cuh", "a") as f:
        f.write("\nstatic const int edited = 1;\n")
    assert bench.kernel_src_hash("attn_fwd_kernel") != h0
