"""Sparse main attention over the selected positions (fp64 oracle) -- TEST INFRASTRUCTURE.

Stage 2 of DSA ("03 long context", section "The Architectural Answer: Read
Less of the Past"): after the indexer's top-k, exact MLA attention is
computed only over the k selected entries.  In the absorbed MLA form the
cached latent row c[s] (576 elements: 512 latent + 64 rotary, bf16, 1,152 B
per token in the same lecture's "Derivation 6") serves as the key of every
query head, and its first 512 elements serve as the value; the per-head cost
per selected entry is 576 + 512 multiply-adds, as that section's FLOP count
128 x (576 + 512) x 2 states.  The kernel layer (same lecture, "Sparsity Is a
Systems Feature: The Blast Radius", "Kernel layer") gathers the selected
entries by token index.

For query t, head h and the selected set S_t (the entries of idx[t] that are
>= 0):

    logit(t, h, s) = scale * sum_d q[t, h, d] * c[s, d]          d < 576
    lse(t, h)      = log sum_{s in S_t} exp(logit(t, h, s))
    o(t, h, :)     = sum_{s in S_t} exp(logit(t, h, s) - lse(t, h)) * c[s, :512]

An empty S_t gives o = 0 and lse = -inf.  The log-sum-exp output lets
attention over disjoint selected sets be combined exactly by the
online-softmax rule (the ring-attention merge in "Teamwork First: Ring
Attention for the Giant Prefill").  The pages do not give the softmax scale;
it is an argument (default 1 / sqrt(576)).

Everything is evaluated in float64 from the stored bytes.
"""

from __future__ import annotations

import numpy as np

LATENT = 576      # elements of a cached latent row (keys)
VALUE = 512       # leading elements that serve as the value


def default_scale(d_qk: int = LATENT) -> float:
    return 1.0 / np.sqrt(d_qk)


def sparse_attention(q: np.ndarray, latent: np.ndarray, idx: np.ndarray, scale: float,
                     d_v: int = VALUE) -> tuple[np.ndarray, np.ndarray]:
    """q [T, H, D] and latent [N, D] (float64), idx [T, k] int (-1 = unused)
    -> (o [T, H, d_v], lse [T, H]) float64."""
    q = np.asarray(q, dtype=np.float64)
    latent = np.asarray(latent, dtype=np.float64)
    idx = np.asarray(idx)
    T, H, D = q.shape
    N = latent.shape[0]
    assert latent.shape[1] == D and d_v <= D
    o = np.zeros((T, H, d_v), dtype=np.float64)
    lse = np.full((T, H), -np.inf, dtype=np.float64)
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        assert np.all(sel < N), "selected position outside the latent cache"
        if sel.size == 0:
            continue
        rows = latent[sel]                              # [n, D] gathered entries
        logits = scale * (q[t] @ rows.T)                # [H, n]
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        den = e.sum(axis=1, keepdims=True)
        lse[t] = (m + np.log(den))[:, 0]
        o[t] = (e / den) @ rows[:, :d_v]
    return o, lse


def merge_partials(o_a: np.ndarray, lse_a: np.ndarray, o_b: np.ndarray, lse_b: np.ndarray):
    """Attention over S_a and over a disjoint S_b -> attention over their union
    (the online-softmax combination: weights exp(lse_x - lse) for each part)."""
    lse = np.logaddexp(lse_a, lse_b)
    with np.errstate(invalid="ignore"):
        wa = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - lse))
        wb = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - lse))
    return wa[..., None] * o_a + wb[..., None] * o_b, lse
