"""The cubic 2^f used on the FMA pipe (CPU check of its error bound and of the
coefficients compiled into the kernels).

The polynomial replaces part of the hardware exponentials in the prefill
softmax; its result is rounded to bf16 (relative spacing 2^-8), so the bound
asked here (1e-4 relative on [-0.5, 0.5]) leaves two orders of margin.  The
header's constants must be the ones the committed fit produces.
"""

import os
import re

import numpy as np

from attention_yarn_rope_b200.exp2_poly import fit, max_rel_error

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_coeffs():
    src = open(os.path.join(ROOT, "attention_yarn_rope_b200", "csrc", "sm100_ptx.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", src).group(1)) for i in range(4)]


def test_header_matches_fit():
    c = fit()
    np.testing.assert_array_equal(np.asarray(_header_coeffs(), np.float32), c)


def test_error_bound():
    assert max_rel_error(_header_coeffs()) < 1e-4


def test_full_range_with_exponent_split():
    # emulate the kernel's split in float32 and compare with exp2 on [-125, 8]
    # (below that the results are denormal, i.e. zero for every later use)
    c = np.asarray(_header_coeffs(), np.float32)
    x = np.linspace(-125.0, 8.0, 400001).astype(np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    p = p.astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4
