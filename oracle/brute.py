"""Brute-force restatements for tiny inputs (TEST INFRASTRUCTURE ONLY).

Pure-Python loops over Python floats (IEEE doubles); used to pin the C oracle.
Nothing here shares code with ``jssa_oracle.c``.
"""
from __future__ import annotations

import itertools
import math


def topk_by_subsets(scores, k):
    """Top-k as an optimisation over k-subsets.

    Among all k-subsets of range(len(scores)) keep those with the largest score
    sum; of those return the lexicographically smallest sorted index tuple.
    For k >= n the whole range is returned.  With exact arithmetic on the
    given doubles this set equals "sort by (score desc, index asc), keep k":
    every maximal-sum set holds all scores above the k-th value, and the
    lexicographic rule takes the lowest indices among the tied ones.  Sums are
    compared with math.fsum (correctly rounded), so ties are exact ties."""
    n = len(scores)
    if k >= n:
        return list(range(n))
    best_sum, best = None, None
    for comb in itertools.combinations(range(n), k):  # lexicographic order
        s = math.fsum(scores[i] for i in comb)
        if best_sum is None or s > best_sum:
            best_sum, best = s, list(comb)
    return best


def attention_loops(q_rows, K_rows, V_rows, scale):
    """Softmax attention of each query row over (K_rows, V_rows) in plain loops.

    Returns (outputs, lse) with outputs[g][c] and lse[g]."""
    outs, lses = [], []
    for qv in q_rows:
        logits = [scale * math.fsum(a * b for a, b in zip(qv, kr)) for kr in K_rows]
        if not logits:
            outs.append([0.0] * (len(V_rows[0]) if V_rows else 0))
            lses.append(-math.inf)
            continue
        m = max(logits)
        ws = [math.exp(x - m) for x in logits]
        z = math.fsum(ws)
        outs.append([math.fsum(w * vr[c] for w, vr in zip(ws, V_rows)) / z for c in range(len(V_rows[0]))])
        lses.append(m + math.log(z))
    return outs, lses
