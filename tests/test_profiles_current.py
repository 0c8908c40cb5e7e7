"""Every ncu summary under profiles/ names the kernel sources it was captured
on (`src_hash <kernel> <hash>` lines, bench.kernel_src_hash: the code of the
kernel's include closure plus its host launcher, comments removed).  A
summary whose kernel has changed since is stale evidence: this CPU check
fails until it is captured again."""

import glob
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _stamps():
    out = []
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as fh:
            for line in fh:
                if line.startswith("src_hash "):
                    _, kernel, h = line.split()
                    out.append((os.path.basename(path), kernel, h))
    return out


def test_every_summary_is_stamped():
    stamped = {f for f, _, _ in _stamps()}
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        assert os.path.basename(path) in stamped, path


def test_summaries_match_current_sources():
    for f, kernel, h in _stamps():
        assert bench.kernel_src_hash(kernel) == h, f"{f}: {kernel} captured at {h}, sources now differ"
