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


def attention(q_heads, rows, scale, d_v):
    """Sparse attention of one query by loops: q_heads H lists of D floats,
    rows n lists of D floats (the selected latent rows) -> (H lists of d_v
    outputs, H log-sum-exps).  Softmax as written: exp of each scaled logit
    over the sum of them all (no max subtraction; fine for tiny inputs)."""
    outs, lses = [], []
    for qh in q_heads:
        if not rows:
            outs.append([0.0] * d_v)
            lses.append(-math.inf)
            continue
        weights = []
        for row in rows:
            dot = 0.0
            for j in range(len(row)):
                dot += qh[j] * row[j]
            weights.append(math.exp(scale * dot))
        total = sum(weights)
        out = [0.0] * d_v
        for w, row in zip(weights, rows):
            for c in range(d_v):
                out[c] += (w / total) * row[c]
        outs.append(out)
        lses.append(math.log(total))
    return outs, lses
