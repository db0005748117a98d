"""Lightning-indexer scores and causal eligibility (fp64 oracle).

Score of key position s for query t ("03 long context", section "The
Architectural Answer: Read Less of the Past", stage 1; "Latent Sparse
Attention", section "Where the time goes"):

    score(t, s) = sum_h  w[t, h] * max(0, sum_d q[t, h, d] * k[s, d])

with H query heads sharing one key per position (MQA-style) and per-head
weights w.  Everything is evaluated in float64 from the stored bytes.

Eligibility under stride-m compression (LeanSparse podcast transcript,
02:36-02:56: CSA keeps one compressed entry per 4 tokens): entry s covers
tokens m*s .. m*s + m - 1 and becomes visible to the query at token position t
once its block is complete, m*s + m - 1 <= t, so query t sees the prefix
s < floor((t + 1) / m).  The pages only say "eligible"; this block-complete
reading is the one adopted.
"""

from __future__ import annotations

import numpy as np


def indexer_scores(q: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """q [T, H, d], w [T, H], keys [N, d] (all float64) -> scores [T, N] float64."""
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    T, H, d = q.shape
    N = keys.shape[0]
    out = np.empty((T, N), dtype=np.float64)
    for t in range(T):
        dots = keys @ q[t].T               # [N, H]: q[t, h] . k[s]
        out[t] = np.maximum(dots, 0.0) @ w[t]   # sum_h w[t, h] * ReLU(.)
    return out


def eligible_count(q_pos: np.ndarray, stride: int, n_keys: int) -> np.ndarray:
    """Number of compressed entries visible to each query position (a prefix)."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    return np.minimum((q_pos + 1) // stride, n_keys)


def eligible_blocks(t: int, stride: int, n_keys: int) -> list:
    """Eligible entries listed one by one: build each block's token range and
    keep the blocks whose every token is at or before t."""
    out = []
    for s in range(n_keys):
        tokens = range(stride * s, stride * s + stride)
        if all(tok <= t for tok in tokens):
            out.append(s)
    return out
