"""Pure-Python brute force for tiny inputs (independent of numpy's BLAS).

Used only to pin the vectorised oracle: every score is a double loop over heads
and dimensions in Python floats, every selection a full ``sorted`` of all
candidates.  The formula and the order are those stated in ``oracle.indexer``
and ``oracle.select``.
"""

from __future__ import annotations

import math


def score(qt, wt, key):
    """qt: H lists of d floats, wt: H floats, key: d floats -> float."""
    total = 0.0
    for h in range(len(qt)):
        dot = 0.0
        for j in range(len(key)):
            dot += qt[h][j] * key[j]
        total += wt[h] * (dot if dot > 0.0 else 0.0)
    return total


def full_sort(values, positions):
    """All candidates sorted by (value desc, position asc), NaN last."""
    def keyf(i):
        v = values[i]
        isnan = v != v
        return (1 if isnan else 0, 0.0 if isnan else -v, positions[i])
    order = sorted(range(len(values)), key=keyf)
    return [positions[i] for i in order], [values[i] for i in order]


def topk(values, positions, k):
    pos, val = full_sort(values, positions)
    pos, val = pos[:k], val[:k]
    while len(pos) < k:
        pos.append(-1)
        val.append(-math.inf)
    return pos, val
