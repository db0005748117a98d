"""Parity of the sparse main attention (CUDA, through the C ABI) with the fp64 oracle.

Tolerance, from the arithmetic: each logit is an fp32 sum of 576 exact
products of bf16 values (relative error a few 1e-7 of the sum of magnitudes),
the weights come from fp32 exp and one division (a few ulp), and each output
is an fp32 weighted sum of at most a few thousand bf16 values (with the
online rescaling, one more rounding per chunk of 64).  Every error term is
below 1e-5 of the largest value magnitude among the selected rows for these
inputs (logits of standard deviation about 2), so the bound checked is
|o - o_ref| <= 1e-4 * max |value| of the query's selected rows and
|lse - lse_ref| <= 1e-4 * (1 + |lse_ref|).  A missed or doubled row moves an
output by about its weight (>= 1e-3 here), a wrong scale or value slice far
more.

Groups of 128 heads over at most 512 slots run on the tensor cores, where
the weights enter the value contraction rounded to bf16 (relative error at
most 2^-9 each; dividing by the sum of the rounded weights keeps them a
convex combination, so each weight is off by at most 2 * 2^-9 of itself):
there the output bound is |o - o_ref| <= 2^-8 * max |value|, and, sharper,
within 2e-3 * max |value| of the same attention with the oracle's weights
rounded to bf16 (fp32 logits can move a weight across a rounding boundary).
lse keeps the 1e-4 bound (it is computed from the unrounded fp32 weights).
"""

import functools

import numpy as np
import pytest
import torch

from oracle.attention import default_scale, merge_partials, sparse_attention
from oracle.formats import bf16_to_f64
from parity_util import dev, dev_bf16
from workloads import get_workload, make_workload
from workloads.synth import make_attention, make_decode

pytestmark = pytest.mark.gpu

ATTN_TOL = 1e-4
ATTN_TOL_TC = 2.0 ** -8
ATTN_TOL_TC_EMUL = 2e-3


def _on_tensor_cores(H, k):
    return H % 128 == 0 and k <= 512


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_lightning_b200 import build as b
    b.build()
    import sparse_attention_indexer_lightning_b200 as lib
    return lib


@functools.lru_cache(maxsize=None)
def data(name):
    return make_workload(name)


def _bf16_weight_attention(q, lat, gidx, scale):
    """The attention with each weight exp(logit - max) rounded to fp32 and then
    to bf16 (nearest even) before the weighted sum and its normalisation:
    the tensor-core kernel's rounding applied to the fp64 logits (test-side
    emulation, not the oracle)."""
    out = np.zeros((q.shape[0], q.shape[1], 512))
    for t in range(q.shape[0]):
        sel = gidx[t][gidx[t] >= 0]
        if sel.size == 0:
            continue
        c = lat[sel]
        lg = scale * (q[t] @ c.T)
        p = np.exp(lg - lg.max(axis=1, keepdims=True)).astype(np.float32)
        pb = (torch.from_numpy(p).to(torch.bfloat16).to(torch.float64)).numpy()
        out[t] = (pb @ c[:, :512]) / pb.sum(axis=1, keepdims=True)
    return out


def _check(out, lse, q_bits, lat_bits, gidx, scale, rows=None, what=""):
    """Compare queries `rows` (all by default) of the GPU result with the oracle;
    gidx holds latent row ids (-1 = unused).  The tolerance follows the path
    the call took (see the module docstring)."""
    rows = range(q_bits.shape[0]) if rows is None else rows
    rows = list(rows)
    tc = _on_tensor_cores(q_bits.shape[1], gidx.shape[1])
    tol = ATTN_TOL_TC if tc else ATTN_TOL
    ro, rl = sparse_attention(bf16_to_f64(q_bits[rows]), bf16_to_f64(lat_bits), gidx[rows], scale)
    re = _bf16_weight_attention(bf16_to_f64(q_bits[rows]), bf16_to_f64(lat_bits), gidx[rows], scale) if tc else None
    for i, t in enumerate(rows):
        sel = gidx[t][gidx[t] >= 0]
        if sel.size == 0:
            assert np.all(out[t] == 0.0), f"{what} t={t}: empty selection must give zeros"
            assert np.all(np.isneginf(lse[t])), f"{what} t={t}: empty selection must give lse = -inf"
            continue
        vmax = np.abs(bf16_to_f64(lat_bits[sel, :512])).max()
        err = np.abs(out[t] - ro[i]).max()
        assert err <= tol * vmax, f"{what} t={t}: output error {err:.3e} > {tol * vmax:.3e}"
        if tc:
            err = np.abs(out[t] - re[i]).max()
            assert err <= ATTN_TOL_TC_EMUL * vmax, f"{what} t={t}: error {err:.3e} against bf16 weights"
        lerr = np.abs(lse[t] - rl[i])
        assert np.all(lerr <= ATTN_TOL * (1 + np.abs(rl[i]))), f"{what} t={t}: lse error {lerr.max():.3e}"


def _run(L, d, scale=None, idx=None, row_off=None):
    idx = d["idx"] if idx is None else idx
    out, lse = L.ls_sparse_attention(dev_bf16(d["q"]), dev_bf16(d["latent"]), dev(idx.astype(np.int32)),
                                     scale=scale, row_off=None if row_off is None else dev(row_off))
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def test_sparse_attention_small(L):
    """7 queries x 16 heads over 300 slots (5 chunks, the last ragged): empty,
    one-row and ragged selections; the unused slots at the tail, then scattered."""
    d = data("attn_s")
    out, lse = _run(L, d)
    _check(out, lse, d["q"], d["latent"], d["idx"], default_scale(), what="attn_s")
    rng = np.random.default_rng(3)
    idx = np.stack([rng.permutation(r) for r in d["idx"]])
    out2, lse2 = _run(L, d, idx=idx)
    _check(out2, lse2, d["q"], d["latent"], idx, default_scale(), what="scattered")


def test_sparse_attention_shapes(L):
    """k = 1, k = 1000 with a larger scale, k = 2048 and 4612 (the LSA read
    list: 4 sinks, a 512-key window, 4096 long-range keys), many heads."""
    for T, H, N, k, scale in ((3, 8, 100, 1, 0.5), (2, 8, 5000, 1000, 0.2), (2, 8, 5000, 2048, None),
                              (2, 8, 9000, 4612, None), (2, 128, 5000, 512, None), (1, 24, 700, 130, 0.05)):
        d = make_attention(T, H, N, k, seed=T * 1000 + k)
        out, lse = _run(L, d, scale=scale)
        _check(out, lse, d["q"], d["latent"], d["idx"], default_scale() if scale is None else scale,
               what=f"T={T} H={H} k={k}")


def test_sparse_attention_row_offsets_and_bad_rows(L):
    """row = idx + row_off[t]; rows outside the cache are skipped and flagged."""
    d = data("attn_s")
    N = d["latent"].shape[0]
    idx = np.where(d["idx"] >= 0, d["idx"] % 1000, -1).astype(np.int32)
    off = np.array([0, 10, 2000, 1500, 0, 2999, 5], dtype=np.int64)
    L.ls_device_status()
    out, lse = _run(L, d, scale=0.07, idx=idx, row_off=off)
    flags = L.ls_device_status()
    g = np.where(idx >= 0, idx + off[:, None], -1)
    bad = (idx >= 0) & (g >= N)
    assert bad.any()
    assert flags & 2        # LS_FAULT_BAD_INDEX
    g = np.where(bad, -1, g)
    _check(out, lse, d["q"], d["latent"], g, 0.07, what="row_off")


def test_sparse_attention_lse_merges_disjoint_parts(L):
    """Attention over the first and the last slots separately, merged by their
    lse (online softmax), equals attention over all of them."""
    d = make_attention(4, 16, 4000, 512, seed=11)
    out, lse = _run(L, d)
    a = d["idx"].copy()
    a[:, 200:] = -1
    b = d["idx"].copy()
    b[:, :200] = -1
    oa, la = _run(L, d, idx=a)
    ob, lb = _run(L, d, idx=b)
    om, lm = merge_partials(oa.astype(np.float64), la.astype(np.float64), ob.astype(np.float64),
                            lb.astype(np.float64))
    vmax = np.abs(bf16_to_f64(d["latent"][:, :512])).max()
    assert np.abs(om - out).max() <= ATTN_TOL * vmax
    assert np.all(np.abs(lm - lse) <= ATTN_TOL * (1 + np.abs(lse)))


def test_attention_merge_kernel(L):
    """ls_attention_merge against the oracle's online-softmax rule on random
    parts, with empty parts (lse = -inf) mixed in and one row empty in every part."""
    rng = np.random.default_rng(5)
    S, T, H, dv = 4, 3, 16, 512
    o = rng.standard_normal((S, T, H, dv)).astype(np.float32)
    lse = (rng.standard_normal((S, T, H)) * 3).astype(np.float32)
    lse[1, 0, :] = -np.inf
    lse[:, 2, 5] = -np.inf
    o[:, 2, 5] = 0.0
    mo, ml = L.ls_attention_merge(dev(o), dev(lse))
    torch.cuda.synchronize()
    mo, ml = mo.cpu().numpy(), ml.cpu().numpy()
    ro, rl = o[0].astype(np.float64), lse[0].astype(np.float64)
    for s in range(1, S):
        ro, rl = merge_partials(ro, rl, o[s].astype(np.float64), lse[s].astype(np.float64))
    assert np.all(mo[2, 5] == 0.0) and np.isneginf(ml[2, 5])
    assert np.abs(mo - ro).max() <= 1e-5 * np.abs(o).max()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(ml), np.isneginf(rl))
    assert np.all(np.abs(ml[fin] - rl[fin]) <= 1e-5 * (1 + np.abs(rl[fin])))


def test_sparse_attention_history_shards_merge(L):
    """The latent rows split into 3 contiguous shards (one per GPU in a
    history-sharded decode): each shard attends over the selected rows it
    holds (row_off = -its first row; other shards' rows are skipped without
    the fault), and ls_attention_merge combines the (o, lse) parts into the
    attention over the whole selection."""
    d = data("attn_s")
    N = d["latent"].shape[0]
    T = d["q"].shape[0]
    q, idx = dev_bf16(d["q"]), dev(d["idx"])
    full_o, full_l = _run(L, d)
    L.ls_device_status()
    parts_o, parts_l = [], []
    for base, length in L.shard_plan(N, 3):
        lat = dev_bf16(np.ascontiguousarray(d["latent"][base:base + length]))
        off = dev(np.full(T, -base, dtype=np.int64))
        o, lse = L.ls_sparse_attention(q, lat, idx, row_off=off, foreign_rows=True)
        parts_o.append(o)
        parts_l.append(lse)
    mo, ml = L.ls_attention_merge(torch.stack(parts_o), torch.stack(parts_l))
    torch.cuda.synchronize()
    assert L.ls_device_status() == 0
    mo, ml = mo.cpu().numpy(), ml.cpu().numpy()
    vmax = np.abs(bf16_to_f64(d["latent"][:, :512])).max()
    assert np.abs(mo - full_o).max() <= ATTN_TOL * vmax
    fin = np.isfinite(full_l)
    assert np.array_equal(np.isneginf(ml), np.isneginf(full_l))
    assert np.all(np.abs(ml[fin] - full_l[fin]) <= ATTN_TOL * (1 + np.abs(full_l[fin])))


def test_sparse_attention_after_decode_selection(L):
    """The decode indexer's top-512 of each sequence, fed as is to the sparse
    attention over a cache holding every sequence's latent rows (row_off =
    b * N): the two stages chained as DSA runs them."""
    wl = get_workload("decode_s")
    dd = make_decode(wl.B, wl.N, seed=wl.seed, ragged=wl.ragged)
    idx, _ = L.ls_decode_select(dev_bf16(dd["q"]), dev(dd["w"]), dev_bf16(dd["k"]), k=wl.k,
                                n_valid=dev(dd["n_valid"]))
    att = make_attention(wl.B, 128, wl.B * wl.N, 1, seed=21)
    off = (np.arange(wl.B, dtype=np.int64) * wl.N)
    out, lse = L.ls_sparse_attention(dev_bf16(att["q"]), dev_bf16(att["latent"]), idx, row_off=dev(off))
    torch.cuda.synchronize()
    sel = idx.cpu().numpy()
    assert np.all((sel >= 0).sum(axis=1) == np.minimum(dd["n_valid"], wl.k))
    g = np.where(sel >= 0, sel + off[:, None], -1)
    _check(out.cpu().numpy(), lse.cpu().numpy(), att["q"], att["latent"], g, default_scale(), what="chained")


def test_sparse_attention_over_lsa_read_lists(L):
    """The LSA flat search's read lists (sinks, the window, the long-range
    keys of the picked buckets, -1 after the row's count) fed as is to the
    sparse attention over a latent cache of the sequence's tokens."""
    wl = get_workload("lsa_flat_s")
    d = data("lsa_flat_s")
    ex = wl.extra
    keys, n = L.ls_lsa_flat_select(dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]),
                                   dev(d["bucket_off"]), dev(d["bucket_mem"]), block_keys=ex["block_keys"],
                                   buckets_per_block=ex["bpb"], n_sink=ex["n_sink"], top_p=wl.top_p,
                                   budget=wl.budget)[:2]
    T = keys.shape[0]
    att = make_attention(T, 16, wl.N, 1, seed=31)
    out, lse = L.ls_sparse_attention(dev_bf16(att["q"]), dev_bf16(att["latent"]), keys)
    torch.cuda.synchronize()
    sel = keys.cpu().numpy()
    nn = n.cpu().numpy()
    assert np.all((sel >= 0).sum(axis=1) == nn) and nn.max() > ex["n_sink"]
    _check(out.cpu().numpy(), lse.cpu().numpy(), att["q"], att["latent"], sel, default_scale(), what="lsa")


@pytest.mark.slow
def test_sparse_attention_full_size_sampled(L):
    """64 decode queries x 128 heads, 512 rows each of a 262144-row cache
    (302 MB): every output finite, sampled queries against the oracle."""
    d = data("attn_decode")
    out, lse = _run(L, d)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    _check(out, lse, d["q"], d["latent"], d["idx"], default_scale(), rows=[0, 17, 40, 63], what="attn_decode")


def test_sparse_attention_tensor_cores(L):
    """The tensor-core path: 128 and 256 heads, k from 1 to 512 (not multiples
    of the 32- and 64-slot chunks), empty queries, unused slots at the tail and
    scattered, a row offset per query, and attention over two disjoint halves
    merged by their lse."""
    for T, H, N, k, scale in ((3, 128, 3000, 512, None), (2, 128, 700, 1, 0.3), (2, 256, 4000, 300, None),
                              (3, 128, 5000, 33, 0.05), (2, 128, 2000, 97, None)):
        d = make_attention(T, H, N, k, seed=7 * T + k + H)
        idx = d["idx"].copy()
        if T > 2:
            idx[0, :] = -1                                # an empty query
            idx[1, ::3] = -1                              # scattered unused slots
        out, lse = _run(L, d, scale=scale, idx=idx)
        _check(out, lse, d["q"], d["latent"], idx, default_scale() if scale is None else scale,
               what=f"tc T={T} H={H} k={k}")
    d = make_attention(3, 128, 6000, 512, seed=99)
    off = np.array([0, 100, 2500], dtype=np.int64)
    idx = np.where(d["idx"] >= 0, d["idx"] % 3000, -1).astype(np.int32)
    out, lse = _run(L, d, idx=idx, row_off=off)
    _check(out, lse, d["q"], d["latent"], np.where(idx >= 0, idx + off[:, None], -1), default_scale(),
           what="tc row_off")
    a = idx.copy()
    a[:, 200:] = -1
    b = idx.copy()
    b[:, :200] = -1
    oa, la = _run(L, d, idx=a, row_off=off)
    ob, lb = _run(L, d, idx=b, row_off=off)
    om, lm = merge_partials(oa.astype(np.float64), la.astype(np.float64), ob.astype(np.float64),
                            lb.astype(np.float64))
    vmax = np.abs(bf16_to_f64(d["latent"][:, :512])).max()
    assert np.abs(om - out).max() <= 2 * ATTN_TOL_TC * vmax
    assert np.all(np.abs(lm - lse) <= ATTN_TOL * (1 + np.abs(lse)))


def test_sparse_attention_tensor_cores_match_cuda_cores(L):
    """Both kernels on the same 128-head inputs: lse agree to fp32 rounding,
    outputs within the tensor-core bound of each other."""
    d = make_attention(4, 128, 6000, 512, seed=5)
    q, lat, idx = dev_bf16(d["q"]), dev_bf16(d["latent"]), dev(d["idx"])
    ot, lt = L.ls_sparse_attention(q, lat, idx)
    oc, lc = L.ls_sparse_attention(q, lat, idx, cuda_cores=True)
    torch.cuda.synchronize()
    ot, lt, oc, lc = (x.cpu().numpy() for x in (ot, lt, oc, lc))
    vmax = np.abs(bf16_to_f64(d["latent"][:, :512])).max()
    assert np.abs(ot - oc).max() <= ATTN_TOL_TC * vmax
    assert np.all(np.abs(lt - lc) <= ATTN_TOL * (1 + np.abs(lc)))
