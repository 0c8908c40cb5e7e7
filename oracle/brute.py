"""Second, independent formulation in scalar Python loops (tiny shapes only).

It shares nothing with :mod:`oracle.rope` / :mod:`oracle.attention` except
the YaRN frequency table, which is an input here:

* RoPE as complex multiplication.  Half-split pairing (the "duplicated
  angles" remark on the NeMo AutoModel ``gpt_oss.rope_utils`` page) makes
  feature pair (i, i+R) the complex number z = x_i + 1j * x_{i+R}; the
  rotation is z * c * exp(1j * p * inv_freq[i]).
* The sink as an extra logit column: for each query row, append ``sink_h`` to
  the visible logits, take an ordinary softmax over all of them and drop the
  sink's column (the form of the Transformers v4.55.0 "Architecture" remark:
  the sink only adds to the denominator).
"""

from __future__ import annotations

import cmath
import math


def rope_complex(vec, pos, inv_freq, conc):
    """Rotate one head vector ``vec`` (list of D floats) at integer ``pos``."""
    R = len(inv_freq)
    out = list(vec)
    for i in range(R):
        z = complex(vec[i], vec[i + R]) * conc * cmath.exp(1j * pos * inv_freq[i])
        out[i] = z.real
        out[i + R] = z.imag
    return out


def attention_concat_column(q, k, v, sinks, scale, window, seq_bounds, positions, inv_freq=None, conc=1.0):
    """q ``[T][Hq][D]``, k / v ``[T][Hkv][D]`` as nested lists; ``seq_bounds`` a
    list of (start, end) token ranges (one entry for BSHD-with-B=1).  Returns
    ``out[T][Hq][D]`` and the per-row sink share ``share[T][Hq]``."""
    T = len(q)
    Hq = len(q[0])
    Hkv = len(k[0])
    D = len(q[0][0])
    G = Hq // Hkv

    def rot(vec, p):
        return rope_complex(vec, p, inv_freq, conc) if inv_freq is not None else list(vec)

    qr = [[rot(q[t][h], positions[t]) for h in range(Hq)] for t in range(T)]
    kr = [[rot(k[t][g], positions[t]) for g in range(Hkv)] for t in range(T)]
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(T)]
    share = [[0.0] * Hq for _ in range(T)]
    for start, end in seq_bounds:
        for i in range(start, end):
            for h in range(Hq):
                g = h // G
                cols = []
                keys = []
                for j in range(start, i + 1):
                    if window > 0 and (i - j) >= window:
                        continue
                    dot = 0.0
                    for d in range(D):
                        dot += qr[i][h][d] * kr[j][g][d]
                    cols.append(scale * dot)
                    keys.append(j)
                cols.append(sinks[h])  # the sink column
                top = max(cols)
                ex = [math.exp(c - top) if c != -math.inf else 0.0 for c in cols]
                den = sum(ex)
                probs = [e / den for e in ex]
                share[i][h] = probs[-1]
                for p, j in zip(probs[:-1], keys):
                    for d in range(D):
                        out[i][h][d] += p * v[j][g][d]
    return out, share
