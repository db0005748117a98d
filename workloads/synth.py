"""Seeded generators for the indexer workloads.

Every generator draws from ``numpy.random.default_rng(seed)`` in a fixed order
and returns host numpy arrays holding the exact bytes both the CUDA path and the
oracle read:

* bf16 tensors as ``uint16`` bit patterns (fp64 draws rounded to nearest even
  through torch's bf16 cast),
* fp8 e4m3 tensors as ``uint8`` codes (torch's ``float8_e4m3fn`` cast, input
  clipped to +-448 first so nothing becomes NaN),
* int8 tensors as ``int8``, scales and head weights as ``float32``,
* product-quantisation (PQ) compact keys as ``uint8`` codes (32 per key, one
  per 4-dimension sub-vector) with fp16 codebooks as ``uint16`` bit patterns
  [32][256][4], the codebooks trained by k-means on a sample of the keys,
* positions as ``int64`` / ``int32``.

Distributions (all workloads): q, k ~ N(0, 1)/sqrt(d), w ~ N(0, 1)/sqrt(H).

Random numbers only: the scoring and selection arithmetic lives in the oracle
and in the CUDA library, never here.
"""

from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

from .shapes import Workload, get_workload


# --------------------------------------------------------------------------- #
# storage-format encoders (library casts)
# --------------------------------------------------------------------------- #
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64/fp32 array -> bf16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float32).numpy()


def to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Values already divided by their scale -> e4m3 codes (uint8)."""
    x = np.clip(np.asarray(x, dtype=np.float32), -448.0, 448.0)
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def e4m3_codes_to_f32(c: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(c, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy()


def _normal(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    return rng.standard_normal(shape) * scale


# --------------------------------------------------------------------------- #
# product quantisation of the compact keys (LeanSparse podcast transcript,
# 07:12-07:34: compact keys of 32 bytes): 32 sub-vectors of 4 dimensions, 256
# centroids each
# --------------------------------------------------------------------------- #
PQ_M, PQ_K, PQ_SUB = 32, 256, 4


def train_pq_books(x: np.ndarray, rng: np.random.Generator, iters: int = 10) -> np.ndarray:
    """Lloyd k-means per sub-space on the rows of x [n, 128], centroids seeded
    from sample rows (distinct when n >= 256; one draw per sub-space), empty
    clusters keeping their centroid; assignments by fp32 squared distance,
    means in fp64.
    Returns the codebooks rounded to fp16, as bit patterns [32][256][4]."""
    n = x.shape[0]
    xs = np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(n, PQ_M, PQ_SUB).transpose(1, 0, 2))
    c = np.stack([xs[m, rng.choice(n, size=PQ_K, replace=n < PQ_K)] for m in range(PQ_M)])  # [32, 256, 4]
    xt32 = torch.from_numpy(xs.astype(np.float32))
    xt64 = torch.from_numpy(xs)
    for _ in range(iters):
        ct = torch.from_numpy(c.astype(np.float32))
        a = ((ct * ct).sum(-1)[:, None, :] - 2.0 * torch.bmm(xt32, ct.transpose(1, 2))).argmin(-1)  # [32, n]
        cnt = torch.zeros(PQ_M, PQ_K, dtype=torch.float64).scatter_add_(1, a, torch.ones_like(a, dtype=torch.float64))
        sums = torch.zeros(PQ_M, PQ_K, PQ_SUB, dtype=torch.float64).scatter_add_(
            1, a[..., None].expand(-1, -1, PQ_SUB), xt64)
        cnt = cnt.numpy()
        nz = cnt > 0
        c[nz] = sums.numpy()[nz] / cnt[nz][:, None]
    return c.astype(np.float16).view(np.uint16)


def encode_pq(x: np.ndarray, books_bits: np.ndarray) -> np.ndarray:
    """Rows of x [n, 128] -> the index of the nearest fp16 centroid (squared
    Euclidean distance in fp32) per sub-vector: uint8 codes [n, 32].  Runs on
    the GPU when one is present (the codes are an input like any other: both
    the oracle and the CUDA path read the same array)."""
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    books = torch.from_numpy(books_bits.view(np.float16).astype(np.float32)).to(dev)  # [32, 256, 4]
    bt = books.transpose(1, 2).contiguous()                                            # [32, 4, 256]
    cn = (books * books).sum(-1)[:, None, :]                                           # [32, 1, 256]
    n = x.shape[0]
    codes = np.empty((n, PQ_M), dtype=np.uint8)
    step = 1 << 15
    for lo in range(0, n, step):
        xs = torch.from_numpy(np.ascontiguousarray(x[lo: lo + step], dtype=np.float32)).to(dev)
        xs = xs.view(-1, PQ_M, PQ_SUB).transpose(0, 1)                                  # [32, c, 4]
        a = (cn - 2.0 * torch.bmm(xs, bt)).argmin(-1)                                   # [32, c]
        codes[lo: lo + xs.shape[1]] = a.transpose(0, 1).to(torch.uint8).cpu().numpy()
    return codes


# --------------------------------------------------------------------------- #
# decode: B sequences, one query each, bf16 keys
# --------------------------------------------------------------------------- #
def make_decode(
    B: int, N: int, H: int = 32, d: int = 128, seed: int = 0, ragged: int = 0,
    n_valid: Optional[np.ndarray] = None,
) -> Dict[str, np.ndarray]:
    rng = np.random.default_rng(seed)
    q = to_bf16_bits(_normal(rng, (B, H, d), 1.0 / math.sqrt(d)))
    w = _normal(rng, (B, H), 1.0 / math.sqrt(H)).astype(np.float32)
    k = np.empty((B, N, d), dtype=np.uint16)
    for b in range(B):  # per sequence, to bound the fp64 working set
        k[b] = to_bf16_bits(_normal(rng, (N, d), 1.0 / math.sqrt(d)))
    if n_valid is None:
        if ragged:
            n_valid = rng.integers(max(N - ragged, 0), N + 1, size=B)
        else:
            n_valid = np.full(B, N)
    return {"q": q, "w": w, "k": k, "n_valid": np.asarray(n_valid, dtype=np.int32)}


# --------------------------------------------------------------------------- #
# prefill: T queries at consecutive token positions, one history of N keys
# --------------------------------------------------------------------------- #
def quantize_e4m3_rows(x: np.ndarray):
    """Rows of x (last axis) -> (e4m3 codes, fp32 scales): scale = amax / 448
    per row (1.0 for an all-zero row), codes = e4m3(x / scale)."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.abs(x).max(axis=-1)
    sc = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    return to_e4m3_codes(x / sc.astype(np.float64)[..., None]), sc


def make_prefill(
    T: int, N: int, q_pos0: int, H: int = 32, d: int = 128, seed: int = 0, fp8: bool = False
) -> Dict[str, np.ndarray]:
    """bf16 queries and history; with fp8 also their e4m3 forms (q8 with one
    scale per (query, head), k8 with one scale per key) quantised from the
    same values."""
    rng = np.random.default_rng(seed)
    q = to_bf16_bits(_normal(rng, (T, H, d), 1.0 / math.sqrt(d)))
    w = _normal(rng, (T, H), 1.0 / math.sqrt(H)).astype(np.float32)
    k = np.empty((N, d), dtype=np.uint16)
    step = 8192
    for s in range(0, N, step):
        e = min(N, s + step)
        k[s:e] = to_bf16_bits(_normal(rng, (e - s, d), 1.0 / math.sqrt(d)))
    q_pos = (q_pos0 + np.arange(T)).astype(np.int64)
    out = {"q": q, "w": w, "k": k, "q_pos": q_pos}
    if fp8:
        out["q8"], out["q_scale"] = quantize_e4m3_rows(bf16_bits_to_f32(q))
        out["k8"], out["k_scale"] = quantize_e4m3_rows(bf16_bits_to_f32(k))
    return out


# --------------------------------------------------------------------------- #
# two-stage decode: fp8 full keys with planted high scorers, int8 compact keys
# --------------------------------------------------------------------------- #
def make_two_stage(
    B: int, N: int, H: int = 32, d: int = 128, seed: int = 0, plant_frac: float = 0.05,
    plant_cos: float = 0.6, ragged: int = 0, pq: bool = False, pq_sample: int = 8192,
) -> Dict[str, np.ndarray]:
    """Full keys: fp8 e4m3 codes with a per-key fp32 scale amax/448.

    A fraction ``plant_frac`` of positions per sequence (chosen uniformly
    without replacement) is replaced by keys whose direction has cosine
    ``plant_cos`` with a per-sequence query direction u = normalise(sum_h
    max(w_h, 0) q_h); the key keeps the norm of the Gaussian draw it replaces.

    Compact keys: int8 codes of the dequantised full key with a per-key fp32
    scale amax/127, rounded half to even, clamped to +-127.  With ``pq``, also
    PQ codes of the dequantised full keys against codebooks trained on
    ``pq_sample`` keys drawn (after everything above) uniformly from all
    sequences' valid positions.
    """
    rng = np.random.default_rng(seed)
    q = to_bf16_bits(_normal(rng, (B, H, d), 1.0 / math.sqrt(d)))
    w = _normal(rng, (B, H), 1.0 / math.sqrt(H)).astype(np.float32)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    fk = np.empty((B, N, d), dtype=np.uint8)
    fk_scale = np.empty((B, N), dtype=np.float32)
    ck = np.empty((B, N, d), dtype=np.int8)
    ck_scale = np.empty((B, N), dtype=np.float32)
    planted = []
    sin = math.sqrt(max(0.0, 1.0 - plant_cos * plant_cos))
    for b in range(B):
        g = _normal(rng, (N, d), 1.0 / math.sqrt(d))
        n_plant = int(round(plant_frac * N))
        pos = np.sort(rng.choice(N, size=n_plant, replace=False))
        u = (np.maximum(w[b].astype(np.float64), 0.0)[:, None] * qf[b]).sum(0)
        u /= np.linalg.norm(u)
        z = rng.standard_normal((n_plant, d))
        z -= (z @ u)[:, None] * u[None, :]
        z /= np.linalg.norm(z, axis=1, keepdims=True)
        norms = np.linalg.norm(g[pos], axis=1, keepdims=True)
        g[pos] = norms * (plant_cos * u[None, :] + sin * z)
        planted.append(pos.astype(np.int32))
        amax = np.abs(g).max(axis=1)
        sc = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
        codes = to_e4m3_codes(g / sc.astype(np.float64)[:, None])
        fk[b] = codes
        fk_scale[b] = sc
        deq = e4m3_codes_to_f32(codes).astype(np.float64) * sc.astype(np.float64)[:, None]
        camax = np.abs(deq).max(axis=1)
        cs = np.where(camax > 0, camax / 127.0, 1.0).astype(np.float32)
        ck[b] = np.clip(np.rint(deq / cs.astype(np.float64)[:, None]), -127, 127).astype(np.int8)
        ck_scale[b] = cs
    if ragged:
        n_valid = rng.integers(max(N - ragged, 0), N + 1, size=B)
    else:
        n_valid = np.full(B, N)
    out = {
        "q": q, "w": w, "fk": fk, "fk_scale": fk_scale, "ck": ck, "ck_scale": ck_scale,
        "n_valid": n_valid.astype(np.int32), "planted": planted,
    }
    if pq:
        def deq(b, sel=slice(None)):
            return e4m3_codes_to_f32(fk[b, sel]).astype(np.float64) * fk_scale[b, sel].astype(np.float64)[:, None]
        tot = int(n_valid.sum())
        pick = np.sort(rng.choice(tot, size=min(pq_sample, tot), replace=False))
        starts = np.concatenate([[0], np.cumsum(n_valid)])
        bi = np.searchsorted(starts, pick, side="right") - 1
        sample = np.concatenate([deq(b, pick[bi == b] - starts[b]) for b in range(B) if np.any(bi == b)])
        books = train_pq_books(sample, rng)
        codes = np.empty((B, N, PQ_M), dtype=np.uint8)
        for b in range(B):
            codes[b] = encode_pq(deq(b), books)
        out["pq_codes"] = codes
        out["pq_books"] = books
    return out


# --------------------------------------------------------------------------- #
# bucket search: clusters of keys scattered over positions, centroid = mean
# --------------------------------------------------------------------------- #
def make_bucket(
    T: int, clusters: int, cluster_size: int, H: int = 32, d: int = 128, seed: int = 0,
    noise_rel: float = 0.3, min_size: int = 0, max_size: int = 0,
) -> Dict[str, np.ndarray]:
    """Clustered keys for the bucket search.

    Cluster centres ~ N(0, 1)/sqrt(d); each member = centre + noise whose
    expected norm is ``noise_rel`` times the centre's norm (per-coordinate std
    noise_rel*|c|/sqrt(d)).  Members sit at positions given by a seeded
    permutation, stored in ascending order per bucket (CSR ``bucket_off`` /
    ``bucket_mem``).  The stored centroid is the fp64 mean of the bucket's
    stored bf16 keys, rounded to bf16.  With ``min_size``/``max_size`` set,
    bucket sizes are drawn uniformly from that range instead of being
    ``cluster_size``.
    """
    rng = np.random.default_rng(seed)
    P = clusters
    if min_size and max_size:
        sizes = rng.integers(min_size, max_size + 1, size=P)
    else:
        sizes = np.full(P, cluster_size)
    off = np.zeros(P + 1, dtype=np.int64)
    np.cumsum(sizes, out=off[1:])
    N = int(off[-1])
    centres = _normal(rng, (P, d), 1.0 / math.sqrt(d))
    sigma = noise_rel * np.linalg.norm(centres, axis=1) / math.sqrt(d)
    member_keys = np.repeat(centres, sizes, axis=0) + rng.standard_normal((N, d)) * np.repeat(sigma, sizes)[:, None]
    perm = rng.permutation(N)
    members = np.empty(N, dtype=np.int32)
    keys = np.empty((N, d), dtype=np.uint16)
    kb = to_bf16_bits(member_keys)
    for p in range(P):
        s, e = off[p], off[p + 1]
        order = np.argsort(perm[s:e], kind="stable")
        pos = perm[s:e][order]
        members[s:e] = pos
        keys[pos] = kb[s:e][order]
    kf = bf16_bits_to_f32(keys).astype(np.float64)
    sums = np.add.reduceat(kf[members], off[:-1], axis=0)
    centroids = to_bf16_bits(sums / sizes[:, None])
    q = to_bf16_bits(_normal(rng, (T, H, d), 1.0 / math.sqrt(d)))
    w = _normal(rng, (T, H), 1.0 / math.sqrt(H)).astype(np.float32)
    return {
        "q": q, "w": w, "centroids": centroids, "bucket_off": off.astype(np.int32),
        "bucket_mem": members, "keys": keys,
    }


def make_lsa(
    T: int, L: int, block_keys: int = 512, bpb: int = 64, seed: int = 0, spread: int = 2053, edge: bool = False,
    node_block: int = 4096, fanout: int = 4, levels: int = 1, chunk: bool = False,
) -> Dict[str, np.ndarray]:
    """Native LSA index for one sequence of L tokens and T index queries.

    Complete blocks of ``block_keys`` keys, each cut into pools of 4
    consecutive keys that are grouped into ``bpb`` buckets of 1..4 pools
    (4..16 keys; the grouping stands in for the Ward merges, drawn at random
    here), members stored in ascending position order (CSR ``bucket_off`` /
    ``bucket_mem``, buckets block-major).  Centroids and index queries are
    random 64-d unit vectors rounded to bf16.  Node buckets for the tree
    search, ``levels`` levels of them: every ``node_block`` entries of a level
    (complete blocks only) are grouped ``fanout`` to a node of the level
    above.  Query positions: the last token and every ``spread``-th token
    before it, or (``edge``) the block edges 0, 3, 4, 511, 512, ... followed
    by random positions, or (``chunk``) the last T tokens, one prefill chunk."""
    rng = np.random.default_rng(seed)
    dim = 64
    n_pool = block_keys // 4
    nb = L // block_keys
    P = nb * bpb
    off = np.zeros(P + 1, dtype=np.int64)
    members = np.empty(nb * block_keys, dtype=np.int32)
    at = 0
    bucket_of_rank = np.empty(n_pool, dtype=np.int64)
    for j in range(nb):
        sizes = np.full(bpb, n_pool // bpb)
        for _ in range(3 * bpb // 4):
            a, b = rng.integers(bpb, size=2)
            if a != b and sizes[a] > 1 and sizes[b] < 4:
                sizes[a] -= 1
                sizes[b] += 1
        perm = rng.permutation(n_pool)
        cuts = np.concatenate([[0], np.cumsum(sizes)])
        # bucket i takes the pools perm[cuts[i]:cuts[i+1]], in ascending order
        bucket_of_rank[:] = np.repeat(np.arange(bpb), sizes)
        pools = perm[np.lexsort((perm, bucket_of_rank))]
        pos = (j * block_keys + 4 * pools[:, None] + np.arange(4)[None, :]).reshape(-1)
        members[at:at + pos.size] = pos
        off[j * bpb + 1:(j + 1) * bpb + 1] = at + 4 * cuts[1:]
        at += pos.size
    c = rng.standard_normal((P, dim))
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    q = rng.standard_normal((T, dim))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    # node buckets: a node's centroid is the normalised sum of every key
    # beneath it; the synthetic buckets have no keys, so a bucket's key sum
    # is taken as its size x its (bf16) centroid and a node's as the sum of
    # its children's
    node_levels = []
    ksum = bf16_bits_to_f32(to_bf16_bits(c)).astype(np.float64) * np.diff(off)[:, None].astype(np.float64)
    for _ in range(levels):
        n_up = (ksum.shape[0] // node_block) * (node_block // fanout)
        ksum = ksum[:n_up * fanout].reshape(n_up, fanout, dim).sum(axis=1)
        norms = np.linalg.norm(ksum, axis=1, keepdims=True)
        node_levels.append(to_bf16_bits(ksum / np.where(norms > 0, norms, 1.0)) if n_up
                           else np.zeros((0, dim), dtype=np.uint16))
    if edge:
        fixed = [0, 3, 4, 511, 512, 513, 1023, 1024, 1536, 2047, 2048, L - 1]
        rest = np.sort(rng.integers(0, L, size=max(0, T - len(fixed))))
        q_pos = np.concatenate([fixed, rest])[:T].astype(np.int64)
    elif chunk:
        q_pos = np.arange(L - T, L, dtype=np.int64)
    else:
        q_pos = (L - 1 - spread * np.arange(T)).astype(np.int64)
    return {"q_idx": to_bf16_bits(q), "q_pos": q_pos, "centroids": to_bf16_bits(c),
            "bucket_off": off.astype(np.int32), "bucket_mem": members,
            "node_centroids": node_levels[0] if levels else np.zeros((0, dim), dtype=np.uint16),
            "node_levels": node_levels}


# --------------------------------------------------------------------------- #
# sparse main attention: a latent cache of N rows x d bf16 (d = 576: 512
# latent + 64 rotary elements), T queries of H heads, and per query k slots of
# selected rows (distinct, -1 after the valid prefix)
# --------------------------------------------------------------------------- #
def make_attention(T: int, H: int, N: int, k: int, d: int = 576, seed: int = 0,
                   ragged: int = 0, q_std: float = 2.0 / 24.0) -> Dict[str, np.ndarray]:
    """q ~ N(0, q_std^2) and latent ~ N(0, 1) per element (logits of standard
    deviation about q_std * sqrt(d) before the 1/sqrt(d) scale: 2 by default).
    With ``ragged``, row 0 selects nothing, row 1 one row, the others a valid
    prefix of length in [k - ragged, k]."""
    rng = np.random.default_rng(seed)
    q = to_bf16_bits(_normal(rng, (T, H, d), q_std))
    latent = np.empty((N, d), dtype=np.uint16)
    step = 1 << 16
    for r0 in range(0, N, step):          # in chunks, to bound the fp64 working set
        n = min(step, N - r0)
        latent[r0:r0 + n] = to_bf16_bits(rng.standard_normal((n, d)))
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        if ragged:
            nv = 0 if t == 0 else 1 if t == 1 else int(rng.integers(max(k - ragged, 0), k + 1))
        else:
            nv = k
        nv = min(nv, N)
        idx[t, :nv] = rng.choice(N, size=nv, replace=False)
    return {"q": q, "latent": latent, "idx": idx}


def make_workload(wl, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs for a named workload (or a ``Workload``)."""
    if isinstance(wl, str):
        wl = get_workload(wl)
    assert isinstance(wl, Workload)
    s = wl.seed if seed is None else seed
    if wl.kind == "decode":
        return make_decode(wl.B, wl.N, wl.H, wl.d, s, ragged=wl.ragged)
    if wl.kind == "prefill":
        return make_prefill(wl.T, wl.N, wl.q_pos0, wl.H, wl.d, s, fp8=bool(wl.extra.get("fp8", 0)))
    if wl.kind == "two_stage":
        return make_two_stage(wl.B, wl.N, wl.H, wl.d, s, wl.plant_frac, wl.plant_cos, ragged=wl.ragged,
                              pq=bool(wl.extra.get("pq", 0)))
    if wl.kind == "bucket":
        return make_bucket(
            wl.T, wl.clusters, wl.cluster_size, wl.H, wl.d, s, wl.noise_rel,
            wl.extra.get("min_size", 0), wl.extra.get("max_size", 0),
        )
    if wl.kind == "lsa":
        ex = wl.extra
        return make_lsa(wl.T, wl.N, ex.get("block_keys", 512), ex.get("bpb", 64), s, ex.get("spread", 2053),
                        bool(ex.get("edge", 0)), ex.get("node_block", 4096), ex.get("fanout", 4), ex.get("levels", 1),
                        bool(ex.get("chunk", 0)))
    if wl.kind == "attention":
        return make_attention(wl.T, wl.H, wl.N, wl.k, wl.d, s, ragged=wl.ragged)
    raise ValueError(wl.kind)
