"""Pure-Python brute force of paged decode attention, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Lists of Python
floats and ``math.exp``; no numpy arithmetic.  Same definition as the C
oracle, written independently: logical token ``i`` of a sequence is slot
``i % block_size`` of physical block ``table[i // block_size]`` ("What vLLM
Is and Why It Exists", section "The idea vLLM started from: pages"), and the
output is the softmax-weighted mean of the values.
"""
from __future__ import annotations

import math


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale):
    """``q[s][h][d]``, caches ``[N][Hkv][bs][D]`` as nested lists of floats."""
    S, Hq = len(q), len(q[0])
    Hkv, bs = len(k_cache[0]), len(k_cache[0][0])
    group = Hq // Hkv
    out = []
    for s in range(S):
        n = int(context_lens[s])
        rows = []
        for h in range(Hq):
            D = len(q[s][h])
            if n == 0:
                rows.append([0.0] * D)
                continue
            g = h // group
            keys, vals = [], []
            for i in range(n):
                b = int(block_tables[s][i // bs])
                keys.append(k_cache[b][g][i % bs])
                vals.append(v_cache[b][g][i % bs])
            logits = [scale * math.fsum(a * b for a, b in zip(q[s][h], k)) for k in keys]
            top = max(logits)
            weights = [math.exp(x - top) for x in logits]
            total = math.fsum(weights)
            rows.append([math.fsum(w * v[d] for w, v in zip(weights, vals)) / total
                         for d in range(D)])
        out.append(rows)
    return out
