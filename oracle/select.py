"""Top-k selection and the three search pipelines (fp64 oracle).

Order ("Latent Sparse Attention", section "What the kernels do about the
top-p": a packed key with the score bits above the inverted id, so a higher
score wins and, among equal scores, the lower id):

    score descending, then position ascending.

Readings where the pages are silent: -0.0 and +0.0 are equal scores; NaN ranks
below every number including -inf; the selected list is returned in that
canonical order (the pages leave it unsorted); a row with fewer than k
eligible positions is padded with position -1 and value -inf.

Pipelines:

* decode / prefill selection: exact scores of every eligible position, then
  top-k (k = 512; LeanSparse podcast transcript, 01:33-02:06).
* fp8 prefill selection: the same with e4m3 queries (one fp32 scale per
  query head) and e4m3 keys (one fp32 scale per key), decoded exactly from
  their codes and scaled ("03 long context" lecture, section "Sparsity Is a
  Systems Feature: The Blast Radius": the indexer scores as an FP8 GEMM over
  the 128-dim keys; section "The Architectural Answer: Read Less of the
  Past", stage 1: a 128-dim FP8 key with a 4 B scale).
* two-stage decode search (LeanSparse podcast transcript, 07:12-08:00): scores
  from compact keys, keep a shortlist, score the shortlist's original keys
  exactly, keep the top k of those.
* native LSA flat search ("Latent Sparse Attention", "How LSA finds the keys"
  and "The method, term by term", steps 5-6): score the unit centroid of
  every bucket of the blocks before the query's own with one 64-d dot
  product, keep the top-p buckets, read them best first skipping members
  that fall in the sinks or the window until the budget is held (the last
  bucket cut short); the read list is the sinks, the window (the query's own
  block up to the query) and those long-range keys.
* LSA tree search, one node level ("Latent Sparse Attention", "The tree, step
  by step"): node buckets group 4 buckets of a complete 4096-bucket block;
  the beam keeps the best node buckets, the search steps down to their
  children plus the uncovered buckets and picks the top-p there.  Several
  levels: the beam starts at the lowest level with at most 32768 node
  buckets and steps down one level at a time the same way.
* bucket search ("Latent Sparse Attention", "How LSA finds the keys" and "The
  method, term by term", steps 5-6): score every bucket centroid with the
  indexer score, keep the top-p buckets, read them best first appending their
  members until the budget is held (the last bucket cut short), score those
  keys exactly and keep the top k.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, dequant, pq_decode
from .indexer import eligible_count, indexer_scores


def select_topk(values: np.ndarray, positions: np.ndarray, k: int):
    """Top-k of one candidate list by (value desc, position asc).

    Returns (positions [k] int64, values [k]) padded with (-1, -inf)."""
    values = np.asarray(values)
    positions = np.asarray(positions, dtype=np.int64)
    nan = np.isnan(values)
    v = np.where(nan, 0.0, values).astype(np.float64)
    # np.lexsort: the last key is the primary one.
    order = np.lexsort((positions, -v, nan))
    take = order[:k]
    pos = np.full(k, -1, dtype=np.int64)
    val = np.full(k, -np.inf, dtype=values.dtype if values.dtype.kind == "f" else np.float64)
    pos[: take.size] = positions[take]
    val[: take.size] = values[take]
    return pos, val


def topk_rows(scores: np.ndarray, n_valid, k: int):
    """Row-wise top-k over the prefix [0, n_valid[r]) of each row.

    Works in the dtype of ``scores`` (fp32 arrays are compared as fp32)."""
    scores = np.atleast_2d(scores)
    R, N = scores.shape
    if n_valid is None:
        n_valid = np.full(R, N)
    idx = np.empty((R, k), dtype=np.int64)
    val = np.empty((R, k), dtype=scores.dtype)
    for r in range(R):
        n = int(min(max(int(n_valid[r]), 0), N))
        idx[r], val[r] = select_topk(scores[r, :n], np.arange(n), k)
    return idx, val


# --------------------------------------------------------------------------- #
# pipelines
# --------------------------------------------------------------------------- #
def decode_select(q_bits, w, k_bits, n_valid, k: int = 512, return_scores: bool = False):
    """One query per sequence over bf16 keys: exact scores then top-k."""
    B = q_bits.shape[0]
    idx = np.empty((B, k), dtype=np.int64)
    val = np.empty((B, k), dtype=np.float64)
    all_scores = []
    for b in range(B):
        n = int(n_valid[b]) if n_valid is not None else k_bits.shape[1]
        s = indexer_scores(bf16_to_f64(q_bits[b])[None], np.asarray(w[b], np.float64)[None],
                           bf16_to_f64(k_bits[b, :n]))[0]
        idx[b], val[b] = select_topk(s, np.arange(n), k)
        all_scores.append(s)
    if return_scores:
        return idx, val, all_scores
    return idx, val


def prefill_select(q_bits, w, q_pos, k_bits, stride: int = 4, k: int = 512, rows=None,
                   return_scores: bool = False):
    """Causal prefill selection for the queries in ``rows`` (default: all)."""
    T = q_bits.shape[0]
    N = k_bits.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    n_t = eligible_count(q_pos, stride, N)
    keys = bf16_to_f64(k_bits)
    idx = np.empty((rows.size, k), dtype=np.int64)
    val = np.empty((rows.size, k), dtype=np.float64)
    all_scores = []
    for i, t in enumerate(rows):
        n = int(n_t[t])
        s = indexer_scores(bf16_to_f64(q_bits[t])[None], np.asarray(w[t], np.float64)[None], keys[:n])[0]
        idx[i], val[i] = select_topk(s, np.arange(n), k)
        all_scores.append(s)
    if return_scores:
        return idx, val, all_scores
    return idx, val


def prefill_select_fp8(q8, q_scale, w, q_pos, k8, k_scale, stride: int = 4, k: int = 512, rows=None,
                       return_scores: bool = False):
    """Causal prefill selection with fp8 inputs: query head h of query t is
    e4m3(q8[t, h]) * q_scale[t, h], key n is e4m3(k8[n]) * k_scale[n]; the
    scores and the selection are then those of prefill_select."""
    T = q8.shape[0]
    N = k8.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    n_t = eligible_count(q_pos, stride, N)
    keys = dequant(k8, k_scale, "e4m3")
    idx = np.empty((rows.size, k), dtype=np.int64)
    val = np.empty((rows.size, k), dtype=np.float64)
    all_scores = []
    for i, t in enumerate(rows):
        n = int(n_t[t])
        qt = dequant(q8[t], q_scale[t], "e4m3")          # [H, d]
        s = indexer_scores(qt[None], np.asarray(w[t], np.float64)[None], keys[:n])[0]
        idx[i], val[i] = select_topk(s, np.arange(n), k)
        all_scores.append(s)
    if return_scores:
        return idx, val, all_scores
    return idx, val


def two_stage_pq_select(q_bits, w, pq_codes, pq_books, fk, fk_scale, n_valid, shortlist: int, k: int = 512,
                        rows=None, return_detail: bool = False):
    """The two-stage search with PQ compact keys: scores of the PQ-decoded keys
    -> shortlist -> exact re-rank of the fp8 originals -> top-k."""
    return two_stage_select(q_bits, w, None, None, fk, fk_scale, n_valid, shortlist, k, rows, return_detail,
                            coarse=lambda b, n: pq_decode(pq_codes[b, :n], pq_books))


def two_stage_select(q_bits, w, ck, ck_scale, fk, fk_scale, n_valid, shortlist: int, k: int = 512,
                     rows=None, return_detail: bool = False, coarse=None):
    """Compact scan -> shortlist -> exact re-rank of the originals -> top-k.
    ``coarse(b, n)`` gives the compact keys of row b (default: int8 x scale)."""
    B = q_bits.shape[0]
    rows = np.arange(B) if rows is None else np.asarray(rows)
    idx = np.empty((rows.size, k), dtype=np.int64)
    val = np.empty((rows.size, k), dtype=np.float64)
    detail = []
    for i, b in enumerate(rows):
        n = int(n_valid[b]) if n_valid is not None else fk.shape[1]
        qb = bf16_to_f64(q_bits[b])[None]
        wb = np.asarray(w[b], np.float64)[None]
        kc = dequant(ck[b, :n], ck_scale[b, :n], "int8") if coarse is None else coarse(b, n)
        s_hat = indexer_scores(qb, wb, kc)[0]
        short, _ = select_topk(s_hat, np.arange(n), shortlist)
        short = short[short >= 0]
        exact = indexer_scores(qb, wb, dequant(fk[b, short], fk_scale[b, short], "e4m3"))[0]
        idx[i], val[i] = select_topk(exact, short, k)
        if return_detail:
            detail.append({"s_hat": s_hat, "shortlist": short, "exact_short": exact})
    if return_detail:
        return idx, val, detail
    return idx, val


def expand_buckets(picked, bucket_off, bucket_mem, budget: int) -> np.ndarray:
    """Best-first expansion: members of the picked buckets in pick order, in
    stored order within a bucket, until ``budget`` keys are held."""
    out = []
    for p in picked:
        if p < 0:
            break
        for m in bucket_mem[bucket_off[p]: bucket_off[p + 1]]:
            if len(out) == budget:
                return np.asarray(out, dtype=np.int64)
            out.append(int(m))
    return np.asarray(out, dtype=np.int64)


def bucket_select(q_bits, w, centroids, bucket_off, bucket_mem, key_bits, top_p: int, budget: int,
                  k: int = 512, rows=None, return_detail: bool = False):
    """Centroid scores -> top-p buckets -> expansion -> exact rescore -> top-k."""
    T = q_bits.shape[0]
    P = centroids.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    cent = bf16_to_f64(centroids)
    idx = np.empty((rows.size, k), dtype=np.int64)
    val = np.empty((rows.size, k), dtype=np.float64)
    detail = []
    for i, t in enumerate(rows):
        qt = bf16_to_f64(q_bits[t])[None]
        wt = np.asarray(w[t], np.float64)[None]
        cs = indexer_scores(qt, wt, cent)[0]
        picked, _ = select_topk(cs, np.arange(P), top_p)
        cand = expand_buckets(picked, bucket_off, bucket_mem, budget)
        exact = indexer_scores(qt, wt, bf16_to_f64(key_bits[cand]))[0]
        idx[i], val[i] = select_topk(exact, cand, k)
        if return_detail:
            detail.append({"centroid_scores": cs, "picked": picked, "cand": cand, "exact_cand": exact})
    if return_detail:
        return idx, val, detail
    return idx, val


def lsa_visible(q_pos, block_keys: int, buckets_per_block: int, n_buckets: int) -> np.ndarray:
    """Buckets a query sees: those of the complete blocks before its own."""
    q_pos = np.maximum(np.asarray(q_pos, dtype=np.int64), 0)
    return np.minimum((q_pos // block_keys) * buckets_per_block, n_buckets)


def lsa_read_list(picked, pos: int, bucket_off, bucket_mem, block_keys: int, n_sink: int, budget: int) -> np.ndarray:
    """The keys a query at position ``pos`` reads, given its picked buckets in
    pick order: the sinks below its window, the window (its own block up to
    ``pos``), then the picked buckets' members in pick order and stored order,
    members that fall in the sinks or the window skipped, until ``budget``
    long-range keys are held."""
    pos = max(int(pos), 0)
    wstart = (pos // block_keys) * block_keys
    sinks = [s for s in range(n_sink) if s < wstart]
    window = list(range(wstart, pos + 1))
    longr = []
    for p in picked:
        if p < 0 or len(longr) == budget:
            break
        for m in bucket_mem[bucket_off[p]: bucket_off[p + 1]]:
            m = int(m)
            if m < n_sink or m >= wstart:
                continue
            if len(longr) == budget:
                break
            longr.append(m)
    return np.asarray(sinks + window + longr, dtype=np.int64)


def lsa_flat_select(q_idx_bits, q_pos, centroid_bits, bucket_off, bucket_mem, block_keys: int,
                    buckets_per_block: int, n_sink: int, top_p: int, budget: int, rows=None,
                    return_detail: bool = False):
    """Read lists of the native LSA flat search, one per query (``rows``,
    default all)."""
    T = q_idx_bits.shape[0]
    P = centroid_bits.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    cent = bf16_to_f64(centroid_bits)
    vis = lsa_visible(q_pos, block_keys, buckets_per_block, P)
    out, detail = [], []
    for t in rows:
        v = int(vis[t])
        scores = cent[:v] @ bf16_to_f64(q_idx_bits[t])          # one dot product per visible bucket
        picked, _ = select_topk(scores, np.arange(v), top_p)
        out.append(lsa_read_list(picked, q_pos[t], bucket_off, bucket_mem, block_keys, n_sink, budget))
        detail.append({"scores": scores, "picked": picked, "visible": v})
    if return_detail:
        return out, detail
    return out


def lsa_tree_select(q_idx_bits, q_pos, centroid_bits, node_bits, bucket_off, bucket_mem, block_keys: int,
                    buckets_per_block: int, node_block: int, fanout: int, beam: int, n_sink: int, top_p: int,
                    budget: int, rows=None, return_detail: bool = False):
    """Read lists of the LSA tree search with one level of node buckets
    ("Latent Sparse Attention", "The tree, step by step"): score the node
    buckets of the complete node blocks among the query's visible buckets,
    keep the best ``beam``, step down to their children plus the visible
    buckets no node covers, pick the top-p of those, read them."""
    T = q_idx_bits.shape[0]
    P = centroid_bits.shape[0]
    P1 = node_bits.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    cent = bf16_to_f64(centroid_bits)
    nodes = bf16_to_f64(node_bits)
    vis = lsa_visible(q_pos, block_keys, buckets_per_block, P)
    out, detail = [], []
    for t in rows:
        v = int(vis[t])
        vn = min((v // node_block) * (node_block // fanout), P1)
        qv = bf16_to_f64(q_idx_bits[t])
        node_scores = nodes[:vn] @ qv
        kept, _ = select_topk(node_scores, np.arange(vn), beam)
        kept = kept[kept >= 0]
        cand = [int(n) * fanout + c for n in kept for c in range(fanout)] + list(range(vn * fanout, v))
        cand = np.asarray(cand, dtype=np.int64)
        scores = cent[cand] @ qv if cand.size else np.zeros(0)
        picked, _ = select_topk(scores, cand, top_p)
        out.append(lsa_read_list(picked, q_pos[t], bucket_off, bucket_mem, block_keys, n_sink, budget))
        detail.append({"node_scores": node_scores, "beam": kept, "visible_nodes": vn, "candidates": cand,
                       "scores": scores, "picked": picked, "visible": v})
    if return_detail:
        return out, detail
    return out


def lsa_tree_levels(vis_buckets: int, level_sizes, node_block: int, fanout: int):
    """Visible entries of every level for a query that sees ``vis_buckets``
    buckets: level l's nodes exist for the complete node blocks of level
    l - 1 ("Latent Sparse Attention", "The tree, step by step": every
    node_block entries of a level form a node cluster block, grouped fanout to
    a node of the level above)."""
    v = [int(vis_buckets)]
    for size in level_sizes:
        v.append(min(int(size), (v[-1] // node_block) * (node_block // fanout)))
    return v


def lsa_tree_levels_select(q_idx_bits, q_pos, centroid_bits, level_bits, bucket_off, bucket_mem, block_keys: int,
                           buckets_per_block: int, node_block: int, fanout: int, beam: int, start_nodes: int,
                           n_sink: int, top_p: int, budget: int, rows=None, return_detail: bool = False):
    """Read lists of the LSA tree search over several levels of node buckets
    ("Latent Sparse Attention", "The tree, step by step"): node n of level l
    covers entries fanout*n .. fanout*n + fanout - 1 of level l - 1 (level 0:
    the buckets).  The beam starts at the lowest level with at most
    ``start_nodes`` node buckets (the top level if none has so few) and
    scores every visible node there, keeps the best ``beam``; at each level
    below it scores the kept nodes' children plus the level's visible entries
    no node above covers, keeps the best ``beam`` again; at the bucket level it
    picks the top-p of the last beam's children and the uncovered buckets,
    which are read as in the flat search.  ``level_bits``: the node centroids
    of levels 1..L (bf16 bits), L >= 1."""
    T = q_idx_bits.shape[0]
    P = centroid_bits.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    levels = [centroid_bits] + list(level_bits)
    sizes = [lv.shape[0] for lv in levels]
    L = len(level_bits)
    assert L >= 1
    start = next((lv for lv in range(1, L + 1) if sizes[lv] <= start_nodes), L)
    vis = lsa_visible(q_pos, block_keys, buckets_per_block, P)
    out, detail = [], []
    for t in rows:
        v = lsa_tree_levels(vis[t], sizes[1:], node_block, fanout)
        qv = bf16_to_f64(q_idx_bits[t])
        beams, counts = {}, {}
        for lv in range(start, -1, -1):
            if lv == start:                                  # every visible node of the start level
                cand = np.arange(v[start], dtype=np.int64)
            else:                                            # children of the beam, then the uncovered entries
                cand = np.asarray([fanout * int(n) + c for n in beams[lv + 1] for c in range(fanout)]
                                  + list(range(fanout * v[lv + 1], v[lv])), dtype=np.int64)
            scores = bf16_to_f64(levels[lv][cand]) @ qv if cand.size else np.zeros(0)
            counts[lv] = int(cand.size)
            if lv > 0:
                kept, _ = select_topk(scores, cand, beam)
                beams[lv] = kept[kept >= 0]
            else:
                picked, _ = select_topk(scores, cand, top_p)
        out.append(lsa_read_list(picked, q_pos[t], bucket_off, bucket_mem, block_keys, n_sink, budget))
        detail.append({"start": start, "visible": v, "beams": beams, "counts": counts, "candidates": cand,
                       "scores": scores, "picked": picked})
    if return_detail:
        return out, detail
    return out


def recall_at_k(sel: np.ndarray, ref: np.ndarray) -> float:
    """|S intersect S*| / |S*| averaged over rows (padding ignored)."""
    sel = np.atleast_2d(sel)
    ref = np.atleast_2d(ref)
    tot = 0.0
    for a, b in zip(sel, ref):
        bs = set(int(x) for x in b if x >= 0)
        if not bs:
            tot += 1.0
            continue
        tot += len(bs & set(int(x) for x in a if x >= 0)) / len(bs)
    return tot / len(sel)
