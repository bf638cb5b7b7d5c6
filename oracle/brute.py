"""Scalar pure-Python attention for tiny inputs (math.exp / math.log only).

An independent restatement used to cross-check the NumPy oracle: one query
row at a time, one key at a time, no arrays, no library attention routine.
"""
from __future__ import annotations

import math


def row_attention(qrow, keys, vals, scale, allowed=None):
    """(out list[d], lse) of one query row against keys/vals (lists of lists)."""
    logits = []
    for t, krow in enumerate(keys):
        if allowed is not None and not allowed[t]:
            continue
        dot = 0.0
        for a, b in zip(qrow, krow):
            dot += a * b
        logits.append((dot * scale, t))
    if not logits:
        return [0.0] * len(vals[0]), -math.inf
    m = max(s for s, _ in logits)
    den = 0.0
    num = [0.0] * len(vals[0])
    for s, t in logits:
        e = math.exp(s - m)
        den += e
        for c in range(len(num)):
            num[c] += e * vals[t][c]
    return [x / den for x in num], m + math.log(den)


def merge_two(o1, l1, o2, l2):
    """Compose two states of one row by log-add-exp, written out by hand."""
    if l1 == -math.inf:
        return list(o2), l2
    if l2 == -math.inf:
        return list(o1), l1
    m = max(l1, l2)
    a = math.exp(l1 - m)
    b = math.exp(l2 - m)
    lse = m + math.log(a + b)
    wa = math.exp(l1 - lse)
    wb = math.exp(l2 - lse)
    return [wa * x + wb * y for x, y in zip(o1, o2)], lse
