"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Small workloads span several key tiles and ragged tails and are compared
element by element; the full-size workloads are run in the benchmark's launch
configuration and checked on sampled rows the oracle computes one by one.
"""

import functools

import numpy as np
import pytest
import torch

from oracle.formats import bf16_to_f64, dequant, pq_decode
from oracle.indexer import eligible_count, indexer_scores
from oracle.select import (
    bucket_select, expand_buckets, lsa_flat_select, lsa_read_list, lsa_tree_levels_select, lsa_tree_select,
    recall_at_k, select_topk,
    topk_rows, two_stage_pq_select, two_stage_select,
)
from parity_util import (
    RTOL_BF16, RTOL_FP8, check_scores, check_selection, check_set, dev, dev_bf16, dev_e4m3, f32_bits_equal,
)
from workloads import get_workload, make_workload
from workloads.synth import make_decode

pytestmark = pytest.mark.gpu


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


def _ref_decode_scores(d, b, n=None):
    n = d["k"].shape[1] if n is None else n
    return indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None],
                          bf16_to_f64(d["k"][b, :n]))[0]


# --------------------------------------------------------------------------- #
# top-k given fp32 scores: bit-exact
# --------------------------------------------------------------------------- #
def _adversarial_rows(rng, R, N):
    s = rng.standard_normal((R, N)).astype(np.float32)
    if R > 1:
        s[1] = np.round(s[1] * 4) / 4                 # heavy ties
    if R > 2:
        s[2] = 0.0
        s[2, ::3] = -0.0                              # +-0 ties
    if R > 3:
        s[3, ::5] = np.nan
        s[3, ::7] = -np.inf
    if R > 4:
        s[4] = 1.0                                    # all equal
    if R > 5:
        s[5, :] = -np.inf
        s[5, ::11] = np.nan
    return s


# the last four shapes have more rows than SMs: the two- and four-CTAs-per-SM forms
@pytest.mark.parametrize("R,N,k", [(7, 3000, 512), (6, 517, 512), (6, 40000, 4096), (3, 131072, 4096),
                                   (8, 1000, 1), (6, 129, 64), (300, 3000, 512), (300, 20000, 1024),
                                   (160, 9000, 64), (400, 40000, 256)])
def test_topk_bit_exact(L, R, N, k):
    rng = np.random.default_rng(100 + N)
    s = _adversarial_rows(rng, R, N)
    n_valid = rng.integers(0, N + 1, size=R).astype(np.int32)
    n_valid[0] = N
    if R > 6:
        n_valid[6] = 0
    for nv in (None, n_valid):
        idx, val = L.ls_topk_select(dev(s), k, None if nv is None else dev(nv))
        ri, rv = topk_rows(s, nv, k)
        assert np.array_equal(idx.cpu().numpy(), ri), (R, N, k)
        assert f32_bits_equal(val.cpu().numpy(), rv), (R, N, k)


# --------------------------------------------------------------------------- #
# decode scoring and selection
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("name", ["decode_tiny", "decode_s"])
def test_decode_scores_and_select(L, name):
    d = data(name)
    B, H, dd = d["q"].shape
    q = dev_bf16(d["q"])
    w = dev(d["w"])
    k = dev_bf16(d["k"])
    nv = dev(d["n_valid"])
    sc = L.ls_indexer_score(q.view(B, 1, H, dd), w.view(B, 1, H), k, n_valid=nv)[:, 0].cpu().numpy()
    idx, val = L.ls_decode_select(q, w, k, 512, n_valid=nv)
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    for b in range(B):
        n = int(d["n_valid"][b])
        ref = _ref_decode_scores(d, b, n)
        check_scores(sc[b, :n], ref, RTOL_BF16, f"{name} row {b}")
        assert np.all(np.isneginf(sc[b, n:]))
        check_selection(idx[b], val[b], np.arange(n), ref, 512, RTOL_BF16, f"{name} row {b}")
        # selection over the GPU's own scores is bit-exact with the oracle's top-k
        ri, rv = select_topk(sc[b, :n], np.arange(n), 512)
        assert np.array_equal(idx[b], ri) and f32_bits_equal(val[b], rv)


def test_decode_edge_rows(L):
    # rows with no eligible key, fewer than k, exactly k, a ragged final tile
    d = make_decode(B=5, N=700, seed=21, n_valid=np.array([0, 1, 511, 512, 700]))
    q, w, k, nv = dev_bf16(d["q"]), dev(d["w"]), dev_bf16(d["k"]), dev(d["n_valid"])
    idx, val = L.ls_decode_select(q, w, k, 512, n_valid=nv)
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    for b in range(5):
        n = int(d["n_valid"][b])
        ref = _ref_decode_scores(d, b, n) if n else np.zeros(0)
        check_selection(idx[b], val[b], np.arange(n), ref, 512, RTOL_BF16, f"edge row {b}")


@pytest.mark.slow
def test_decode_batch_full_size_sampled(L):
    d = data("decode_batch")
    B, H, dd = d["q"].shape
    q, w, k = dev_bf16(d["q"]), dev(d["w"]), dev_bf16(d["k"])
    idx, val = L.ls_decode_select(q, w, k, 512)
    sc = L.ls_indexer_score(q.view(B, 1, H, dd), w.view(B, 1, H), k)[:, 0]
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    for b in (0, 31, 63):
        ref = _ref_decode_scores(d, b)
        check_scores(sc[b].cpu().numpy(), ref, RTOL_BF16, f"decode_batch row {b}")
        check_selection(idx[b], val[b], np.arange(ref.size), ref, 512, RTOL_BF16, f"decode_batch row {b}")
    # every row: the selection equals the bit-exact top-k of the kernel's own scores
    ri, rv = topk_rows(sc.cpu().numpy(), None, 512)
    assert np.array_equal(idx, ri) and f32_bits_equal(val, rv)


# --------------------------------------------------------------------------- #
# multi-query tiles and converted key formats
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("T", [2, 19, 64])
def test_multiquery_scores_causal(L, T):
    rng = np.random.default_rng(30 + T)
    B, H, dd, N = 2, 32, 128, 900
    from workloads.synth import to_bf16_bits
    qb = to_bf16_bits(rng.standard_normal((B, T, H, dd)) / np.sqrt(dd))
    kb = to_bf16_bits(rng.standard_normal((B, N, dd)) / np.sqrt(dd))
    wv = (rng.standard_normal((B, T, H)) / np.sqrt(H)).astype(np.float32)
    qpos = rng.integers(-2, 4 * N + 8, size=(B, T)).astype(np.int64)
    nv = np.array([N, N - 77], np.int32)
    sc = L.ls_indexer_score(dev_bf16(qb), dev(wv), dev_bf16(kb), n_valid=dev(nv), q_pos=dev(qpos), stride=4)
    sc = sc.cpu().numpy()
    for b in range(B):
        ref = indexer_scores(bf16_to_f64(qb[b]), wv[b].astype(np.float64), bf16_to_f64(kb[b]))
        lim = np.minimum(eligible_count(qpos[b], 4, N), nv[b])
        for t in range(T):
            check_scores(sc[b, t, : lim[t]], ref[t, : lim[t]], RTOL_BF16, f"T={T} b={b} t={t}")
            assert np.all(np.isneginf(sc[b, t, lim[t]:]))


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_converted_key_scores(L, fmt):
    d = data("two_stage_s")
    B, H, dd = d["q"].shape
    q, w = dev_bf16(d["q"]), dev(d["w"])
    if fmt == "int8":
        keys, scale, rtol = dev(d["ck"]), dev(d["ck_scale"]), RTOL_BF16
    else:
        keys, scale, rtol = dev_e4m3(d["fk"]), dev(d["fk_scale"]), RTOL_BF16
    nv = dev(d["n_valid"])
    sc = L.ls_indexer_score(q.view(B, 1, H, dd), w.view(B, 1, H), keys, key_scale=scale, n_valid=nv)[:, 0]
    sc = sc.cpu().numpy()
    codes = d["ck"] if fmt == "int8" else d["fk"]
    scales = d["ck_scale"] if fmt == "int8" else d["fk_scale"]
    for b in range(B):
        n = int(d["n_valid"][b])
        kv = dequant(codes[b, :n], scales[b, :n], fmt)
        ref = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None], kv)[0]
        check_scores(sc[b, :n], ref, rtol, f"{fmt} row {b}")
        assert np.all(np.isneginf(sc[b, n:]))


# --------------------------------------------------------------------------- #
# prefill: streamed history, causal eligibility
# --------------------------------------------------------------------------- #
def _prefill_run(L, d, wl, use_copy_stream=True, full_scores=False):
    T = d["q"].shape[0]
    q, w, qp = dev_bf16(d["q"]), dev(d["w"]), dev(d["q_pos"])
    hist = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    buf0 = torch.empty((wl.tile_keys, 128), dtype=torch.bfloat16, device="cuda")
    buf1 = torch.empty_like(buf0)
    cs = torch.cuda.Stream() if use_copy_stream else None
    idx, val = L.ls_prefill_select_stream(q, w, qp, hist, buf0, buf1, k=wl.k, stride=wl.stride,
                                          tile_keys=wl.tile_keys, full_scores=full_scores, copy_stream=cs)
    torch.cuda.synchronize()
    return q, w, qp, idx.cpu().numpy(), val.cpu().numpy()


def test_prefill_stream_small(L):
    wl = get_workload("prefill_s")
    d = data("prefill_s")
    q, w, qp, idx, val = _prefill_run(L, d, wl)
    T, H, dd = d["q"].shape
    N = d["k"].shape[0]
    n_t = eligible_count(d["q_pos"], wl.stride, N)
    keys = bf16_to_f64(d["k"])
    for t in range(T):
        n = int(n_t[t])
        ref = indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], keys[:n])[0]
        check_selection(idx[t], val[t], np.arange(n), ref, wl.k, RTOL_BF16, f"prefill_s t={t}")
    # the streamed result equals scoring the resident history in one call
    sc = L.ls_indexer_score(q.view(1, T, H, dd), w.view(1, T, H), dev_bf16(d["k"])[None], q_pos=qp.view(1, T),
                            stride=wl.stride)[0]
    ri, rv = L.ls_topk_select(sc, wl.k, n_valid=dev(n_t.astype(np.int32)))
    assert np.array_equal(ri.cpu().numpy(), idx) and f32_bits_equal(rv.cpu().numpy(), val)
    # same answer on a single stream, and from the full-matrix form
    *_, idx2, val2 = _prefill_run(L, d, wl, use_copy_stream=False)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    *_, idx3, val3 = _prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx3, idx) and f32_bits_equal(val3, val)


def test_prefill_stream_overflow(L):
    """Queries whose scores rise with position beat their running list with
    every key of every later tile, so they overflow the candidate slots and take
    the full-tile path; the other queries score 0 everywhere (ties go to the
    lower position), so nothing after the first tile enters their lists."""
    from types import SimpleNamespace
    from workloads.synth import to_bf16_bits
    T, H, dd, N, k, stride = 24, 32, 128, 1000, 32, 4
    rng = np.random.default_rng(7)
    u = rng.standard_normal(dd)
    u /= np.linalg.norm(u)
    alpha = np.linspace(0.05, 1.0, N)
    kbits = to_bf16_bits(alpha[:, None] * u[None, :])
    sign = np.where(np.arange(T) < T // 2, 1.0, -1.0)
    qbits = to_bf16_bits(np.broadcast_to(sign[:, None, None] * u[None, None, :], (T, H, dd)).copy())
    w = (np.abs(rng.standard_normal((T, H))) + 0.1).astype(np.float32)
    q_pos = (stride * N - 1 - rng.integers(0, 300, size=T)).astype(np.int64)
    d = {"q": qbits, "w": w, "k": kbits, "q_pos": q_pos}
    wl = SimpleNamespace(k=k, stride=stride, tile_keys=128)
    q, wd, qp, idx, val = _prefill_run(L, d, wl)
    n_t = eligible_count(q_pos, stride, N)
    keys = bf16_to_f64(kbits)
    for t in range(T):
        n = int(n_t[t])
        ref = indexer_scores(bf16_to_f64(qbits[t])[None], w[t].astype(np.float64)[None], keys[:n])[0]
        check_selection(idx[t], val[t], np.arange(n), ref, k, RTOL_BF16, f"overflow t={t}")
    sc = L.ls_indexer_score(q.view(1, T, H, dd), wd.view(1, T, H), dev_bf16(kbits)[None], q_pos=qp.view(1, T),
                            stride=stride)[0]
    ri, rv = L.ls_topk_select(sc, k, n_valid=dev(n_t.astype(np.int32)))
    assert np.array_equal(ri.cpu().numpy(), idx) and f32_bits_equal(rv.cpu().numpy(), val)


@pytest.mark.parametrize("T,N,tile,k", [(1, 2000, 256, 64), (40, 2000, 256, 1100), (9, 300, 512, 32)])
def test_prefill_stream_shapes(L, T, N, tile, k):
    """One query (the one-query scorer's filter form), k above 1024 (the wide
    top-k and 5k-entry merge rows) and a history shorter than one tile: the
    running form, the full-matrix form and the oracle agree."""
    from types import SimpleNamespace
    from workloads.synth import make_prefill
    d = make_prefill(T, N, 4 * N - T - 37, seed=31)
    wl = SimpleNamespace(k=k, stride=4, tile_keys=tile)
    _, _, _, idx, val = _prefill_run(L, d, wl)
    *_, idx2, val2 = _prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    n_t = eligible_count(d["q_pos"], 4, N)
    keys = bf16_to_f64(d["k"])
    for t in range(T):
        n = int(n_t[t])
        ref = indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], keys[:n])[0]
        check_selection(idx[t], val[t], np.arange(n), ref, k, RTOL_BF16, f"shape ({T},{N},{tile},{k}) t={t}")


@pytest.mark.slow
def test_prefill_chunk_full_size_sampled(L):
    wl = get_workload("prefill_chunk")
    d = data("prefill_chunk")
    _, _, _, idx, val = _prefill_run(L, d, wl)
    # the full-matrix form selects the same
    *_, idx2, val2 = _prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    N = d["k"].shape[0]
    n_t = eligible_count(d["q_pos"], wl.stride, N)
    keys = bf16_to_f64(d["k"])
    for t in (0, 1, 2, 3, 1023, 2048, 4093, 4094, 4095):
        n = int(n_t[t])
        ref = indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], keys[:n])[0]
        check_selection(idx[t], val[t], np.arange(n), ref, wl.k, RTOL_BF16, f"prefill t={t}")


def _sharded_prefill_matches(L, name, shard_counts):
    wl = get_workload(name)
    d = data(name)
    N = d["k"].shape[0]
    q, w, qp = dev_bf16(d["q"]), dev(d["w"]), dev(d["q_pos"])
    _, _, _, idx0, val0 = _prefill_run(L, d, wl)
    for S in shard_counts:
        vals, idxs, offs = [], [], []
        for base, length in L.shard_plan(N, S):
            hist = torch.from_numpy(d["k"][base:base + length].view(np.int16)).view(torch.bfloat16).pin_memory()
            buf0 = torch.empty((wl.tile_keys, 128), dtype=torch.bfloat16, device="cuda")
            buf1 = torch.empty_like(buf0)
            i_s, v_s = L.ls_prefill_select_stream(q, w, qp - base * wl.stride, hist, buf0, buf1, k=wl.k,
                                                  stride=wl.stride, tile_keys=wl.tile_keys)
            vals.append(v_s)
            idxs.append(i_s)
            offs.append(base)
        mi, mv = L.ls_merge_select(torch.stack(vals), torch.stack(idxs), dev(np.asarray(offs, dtype=np.int32)),
                                   k=wl.k)
        torch.cuda.synchronize()
        assert np.array_equal(mi.cpu().numpy(), idx0), (name, S)
        assert f32_bits_equal(mv.cpu().numpy(), val0), (name, S)


def test_prefill_sharded_history_merge(L):
    """A history split into S contiguous shards (one per GPU in a sharded
    prefill): each shard's selection for the same queries, positions shifted
    so the causal rule holds per shard, merged by ls_merge_select, equals the
    selection over the whole history bit for bit."""
    _sharded_prefill_matches(L, "prefill_s", (2, 3))


@pytest.mark.slow
def test_prefill_sharded_history_merge_full_size(L):
    """The 4096-query prefill chunk over 32768 keys in 4 and 3 history shards
    (one 8192-key tile each, and ragged shards) merges to the unsharded
    selection bit for bit."""
    _sharded_prefill_matches(L, "prefill_chunk", (4, 3))


def test_merge_select_edge_cases(L):
    """ls_merge_select on hand-made shard lists: one shard (the identity), a
    shard whose lists are all padding, lists shorter than k (fewer
    candidates than k: the result is padded), equal values across shards
    (the lower global position first), compared with the top-k of the union
    of the valid entries."""
    rng = np.random.default_rng(8)
    T, k_in = 6, 40
    for S, k, empty_shard in ((1, 40, None), (3, 40, 1), (2, 100, None), (4, 64, 3)):
        offs = np.array([1000 * s for s in range(S)], dtype=np.int32)
        vals = np.full((S, T, k_in), -np.inf, dtype=np.float32)
        idx = np.full((S, T, k_in), -1, dtype=np.int32)
        for s in range(S):
            for t in range(T):
                n = 0 if s == empty_shard else int(rng.integers(0, k_in + 1))
                pos = np.sort(rng.choice(900, size=n, replace=False))
                v = np.round(rng.standard_normal(n) * 2).astype(np.float32)   # many equal values
                sel_pos, sel_val = select_topk(v, pos, k_in)                   # each list in canonical order
                idx[s, t], vals[s, t] = sel_pos.astype(np.int32), sel_val.astype(np.float32)
        mi, mv = L.ls_merge_select(dev(vals), dev(idx), dev(offs), k=k)
        torch.cuda.synchronize()
        mi, mv = mi.cpu().numpy(), mv.cpu().numpy()
        for t in range(T):
            ok = idx[:, t] >= 0
            gpos = (idx[:, t] + offs[:, None])[ok]
            gval = vals[:, t][ok]
            rp, rv = select_topk(gval, gpos, k)
            assert np.array_equal(mi[t], rp), (S, k, t)
            assert f32_bits_equal(mv[t], rv.astype(np.float32)), (S, k, t)


# --------------------------------------------------------------------------- #
# fp8 indexer: fp8 queries and keys, the prefill streamed from an fp8 history
# --------------------------------------------------------------------------- #
def _fp8_ref(d, t, n):
    qt = dequant(d["q8"][t], d["q_scale"][t], "e4m3")
    return indexer_scores(qt[None], d["w"][t].astype(np.float64)[None],
                          dequant(d["k8"][:n], d["k_scale"][:n], "e4m3"))[0]


def _fp8_prefill_run(L, d, wl, full_scores=False, use_copy_stream=True):
    q8 = dev(d["q8"])
    qs, w, qp = dev(d["q_scale"]), dev(d["w"]), dev(d["q_pos"])
    hk = torch.from_numpy(np.ascontiguousarray(d["k8"])).pin_memory()
    hs = torch.from_numpy(np.ascontiguousarray(d["k_scale"])).pin_memory()
    buf0 = torch.empty(wl.tile_keys * 132, dtype=torch.uint8, device="cuda")
    buf1 = torch.empty_like(buf0)
    cs = torch.cuda.Stream() if use_copy_stream else None
    idx, val = L.ls_prefill_select_stream_fp8(q8, qs, w, qp, hk, hs, buf0, buf1, k=wl.k, stride=wl.stride,
                                              tile_keys=wl.tile_keys, full_scores=full_scores, copy_stream=cs)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy()


def test_fp8_scores(L):
    """Every (query, key) score of a 77-query chunk (a partial last group of 8)
    against 1019 keys (a ragged last tile): within the fp8 tolerance and, since
    the kernel sums exact code products in fp32, within the bf16 one too;
    ineligible keys hold -inf."""
    wl = get_workload("prefill_fp8_s")
    d = data("prefill_fp8_s")
    T, H, dd = d["q8"].shape
    N = d["k8"].shape[0]
    sc = L.ls_indexer_score_fp8(dev(d["q8"])[None], dev(d["q_scale"])[None], dev(d["w"])[None],
                                dev(d["k8"])[None], dev(d["k_scale"])[None], q_pos=dev(d["q_pos"])[None],
                                stride=wl.stride)[0].cpu().numpy()
    n_t = eligible_count(d["q_pos"], wl.stride, N)
    for t in range(T):
        n = int(n_t[t])
        ref = _fp8_ref(d, t, n)
        check_scores(sc[t, :n], ref, RTOL_FP8, f"fp8 scores t={t}")
        check_scores(sc[t, :n], ref, RTOL_BF16, f"fp8 scores (fp32 sums) t={t}")
        assert np.all(np.isneginf(sc[t, n:]))


def test_fp8_scores_batched_n_valid(L):
    """Several problems in one call (B = 3, one query each and a group of 8),
    n_valid cutting each problem's keys."""
    d = data("prefill_fp8_s")
    B, T, N = 3, 9, 300
    rng = np.random.default_rng(5)
    q8 = np.stack([d["q8"][rng.permutation(77)[:T]] for _ in range(B)])
    qs = np.stack([d["q_scale"][:T]] * B)
    w = np.stack([d["w"][b:b + T] for b in range(B)])
    k8 = np.stack([d["k8"][b * 200:b * 200 + N] for b in range(B)])
    ks = np.stack([d["k_scale"][b * 200:b * 200 + N] for b in range(B)])
    nv = np.array([300, 129, 1], dtype=np.int32)
    sc = L.ls_indexer_score_fp8(dev(q8), dev(qs), dev(w), dev(k8), dev(ks), n_valid=dev(nv)).cpu().numpy()
    for b in range(B):
        db = {"q8": q8[b], "q_scale": qs[b], "w": w[b], "k8": k8[b], "k_scale": ks[b]}
        for t in range(T):
            ref = _fp8_ref(db, t, int(nv[b]))
            check_scores(sc[b, t, :nv[b]], ref, RTOL_FP8, f"fp8 batched b={b} t={t}")
            assert np.all(np.isneginf(sc[b, t, nv[b]:]))


def test_fp8_prefill_stream_small(L):
    wl = get_workload("prefill_fp8_s")
    d = data("prefill_fp8_s")
    idx, val = _fp8_prefill_run(L, d, wl)
    T = d["q8"].shape[0]
    N = d["k8"].shape[0]
    n_t = eligible_count(d["q_pos"], wl.stride, N)
    for t in range(T):
        n = int(n_t[t])
        check_selection(idx[t], val[t], np.arange(n), _fp8_ref(d, t, n), wl.k, RTOL_FP8, f"fp8 prefill t={t}")
    # the full-matrix form, a single stream, and scoring the resident history agree bit for bit
    idx2, val2 = _fp8_prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    idx3, val3 = _fp8_prefill_run(L, d, wl, use_copy_stream=False)
    assert np.array_equal(idx3, idx) and f32_bits_equal(val3, val)
    sc = L.ls_indexer_score_fp8(dev(d["q8"])[None], dev(d["q_scale"])[None], dev(d["w"])[None],
                                dev(d["k8"])[None], dev(d["k_scale"])[None], q_pos=dev(d["q_pos"])[None],
                                stride=wl.stride)[0]
    ri, rv = L.ls_topk_select(sc, wl.k, n_valid=dev(n_t.astype(np.int32)))
    assert np.array_equal(ri.cpu().numpy(), idx) and f32_bits_equal(rv.cpu().numpy(), val)


@pytest.mark.parametrize("T,N,tile,k", [(1, 2000, 256, 64), (40, 2000, 256, 1100), (9, 300, 512, 32)])
def test_fp8_prefill_stream_shapes(L, T, N, tile, k):
    """One query (a group of 8 with 7 empty columns), k above 1024, a history
    shorter than one tile: the running form, the full-matrix form and the
    oracle agree."""
    from types import SimpleNamespace
    from workloads.synth import make_prefill
    d = make_prefill(T, N, 4 * N - T - 37, seed=31, fp8=True)
    wl = SimpleNamespace(k=k, stride=4, tile_keys=tile)
    idx, val = _fp8_prefill_run(L, d, wl)
    idx2, val2 = _fp8_prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    n_t = eligible_count(d["q_pos"], 4, N)
    for t in range(T):
        n = int(n_t[t])
        check_selection(idx[t], val[t], np.arange(n), _fp8_ref(d, t, n), k, RTOL_FP8,
                        f"fp8 shape ({T},{N},{tile},{k}) t={t}")


def test_fp8_prefill_stream_overflow(L):
    """Rising scores overflow the candidate slots of half the queries (the
    filter form's overflow path through the full tile); the rest score 0."""
    from types import SimpleNamespace
    from workloads.synth import quantize_e4m3_rows
    T, H, dd, N, k, stride = 24, 32, 128, 1000, 32, 4
    rng = np.random.default_rng(7)
    u = rng.standard_normal(dd)
    u /= np.linalg.norm(u)
    alpha = np.linspace(0.05, 1.0, N)
    k8, ks = quantize_e4m3_rows(alpha[:, None] * u[None, :])
    sign = np.where(np.arange(T) < T // 2, 1.0, -1.0)
    q8, qs = quantize_e4m3_rows(np.broadcast_to(sign[:, None, None] * u[None, None, :], (T, H, dd)).copy())
    w = (np.abs(rng.standard_normal((T, H))) + 0.1).astype(np.float32)
    q_pos = (stride * N - 1 - rng.integers(0, 300, size=T)).astype(np.int64)
    d = {"q8": q8, "q_scale": qs, "w": w, "k8": k8, "k_scale": ks, "q_pos": q_pos}
    wl = SimpleNamespace(k=k, stride=stride, tile_keys=128)
    idx, val = _fp8_prefill_run(L, d, wl)
    idx2, val2 = _fp8_prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    n_t = eligible_count(q_pos, stride, N)
    for t in range(T):
        n = int(n_t[t])
        check_selection(idx[t], val[t], np.arange(n), _fp8_ref(d, t, n), k, RTOL_FP8, f"fp8 overflow t={t}")


@pytest.mark.slow
def test_fp8_prefill_chunk_full_size_sampled(L):
    wl = get_workload("prefill_chunk_fp8")
    d = data("prefill_chunk_fp8")
    idx, val = _fp8_prefill_run(L, d, wl)
    idx2, val2 = _fp8_prefill_run(L, d, wl, full_scores=True)
    assert np.array_equal(idx2, idx) and f32_bits_equal(val2, val)
    N = d["k8"].shape[0]
    n_t = eligible_count(d["q_pos"], wl.stride, N)
    for t in (0, 1, 7, 8, 1023, 2048, 4093, 4094, 4095):
        n = int(n_t[t])
        check_selection(idx[t], val[t], np.arange(n), _fp8_ref(d, t, n), wl.k, RTOL_FP8, f"fp8 prefill t={t}")


# --------------------------------------------------------------------------- #
# two-stage decode search
# --------------------------------------------------------------------------- #
def _check_two_stage(L, name, rows):
    wl = get_workload(name)
    d = data(name)
    q, w = dev_bf16(d["q"]), dev(d["w"])
    if wl.extra.get("pq"):
        books = torch.from_numpy(d["pq_books"].view(np.int16)).view(torch.float16).cuda()
        idx, val, sl = L.ls_decode_two_stage_pq_select(q, w, dev(d["pq_codes"]), books, dev_e4m3(d["fk"]),
                                                       dev(d["fk_scale"]), dev(d["n_valid"]), shortlist=wl.shortlist,
                                                       k=wl.k, want_shortlist=True)
        _, _, det = two_stage_pq_select(d["q"], d["w"], d["pq_codes"], d["pq_books"], d["fk"], d["fk_scale"],
                                        d["n_valid"], wl.shortlist, wl.k, rows=rows, return_detail=True)
    else:
        idx, val, sl = L.ls_decode_two_stage_select(q, w, dev(d["ck"]), dev(d["ck_scale"]), dev_e4m3(d["fk"]),
                                                    dev(d["fk_scale"]), dev(d["n_valid"]), shortlist=wl.shortlist,
                                                    k=wl.k, want_shortlist=True)
        _, _, det = two_stage_select(d["q"], d["w"], d["ck"], d["ck_scale"], d["fk"], d["fk_scale"], d["n_valid"],
                                     wl.shortlist, wl.k, rows=rows, return_detail=True)
    idx, val, sl = idx.cpu().numpy(), val.cpu().numpy(), sl.cpu().numpy()
    recalls = []
    for i, b in enumerate(rows):
        n = int(d["n_valid"][b])
        s_hat = det[i]["s_hat"]
        # shortlist: the band rule on the compact scores (order of the shortlist
        # is the coarse-score order, so its values are not checked here)
        short = sl[b][sl[b] >= 0]
        check_set(sl[b], np.arange(n), s_hat, wl.shortlist, RTOL_BF16, f"{name} shortlist row {b}")
        # final: exact scores of the GPU's shortlist, band rule inside it
        kv = dequant(d["fk"][b, short], d["fk_scale"][b, short], "e4m3")
        exact = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None], kv)[0]
        check_selection(idx[b], val[b], short, exact, wl.k, RTOL_FP8, f"{name} final row {b}")
        # recall against the exact full scan (reported, not pinned)
        kfull = dequant(d["fk"][b, :n], d["fk_scale"][b, :n], "e4m3")
        full = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None], kfull)[0]
        ei, _ = select_topk(full, np.arange(n), wl.k)
        recalls.append(recall_at_k(idx[b][None], ei[None]))
    return recalls


def test_two_stage_small(L):
    rec = _check_two_stage(L, "two_stage_s", [0, 1, 2])
    assert min(rec) > 0.5


@pytest.mark.slow
def test_two_stage_full_size_sampled(L):
    rec = _check_two_stage(L, "two_stage", [0, 17, 31])
    assert min(rec) > 0.5


def test_pq_scores(L):
    wl = get_workload("two_stage_pq_s")
    d = data("two_stage_pq_s")
    books = torch.from_numpy(d["pq_books"].view(np.int16)).view(torch.float16).cuda()
    sc = L.ls_indexer_score_pq(dev_bf16(d["q"]), dev(d["w"]), dev(d["pq_codes"]), books,
                               n_valid=dev(d["n_valid"])).cpu().numpy()
    for b in range(wl.B):
        n = int(d["n_valid"][b])
        ref = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None],
                             pq_decode(d["pq_codes"][b, :n], d["pq_books"]))[0]
        check_scores(sc[b, :n], ref, RTOL_BF16, f"pq row {b}")
        assert np.all(np.isneginf(sc[b, n:]))


def test_two_stage_pq_small(L):
    rec = _check_two_stage(L, "two_stage_pq_s", [0, 1, 2])
    assert min(rec) > 0.5


@pytest.mark.slow
def test_two_stage_pq_full_size_sampled(L):
    rec = _check_two_stage(L, "two_stage_pq", [0, 17, 31])
    assert min(rec) > 0.5


# --------------------------------------------------------------------------- #
# bucket search
# --------------------------------------------------------------------------- #
def _check_bucket(L, name, rows):
    wl = get_workload(name)
    d = data(name)
    q, w = dev_bf16(d["q"]), dev(d["w"])
    idx, val, picked = L.ls_bucket_select(q, w, dev_bf16(d["centroids"]), dev(d["bucket_off"]),
                                          dev(d["bucket_mem"]), dev_bf16(d["keys"]), top_p=wl.top_p,
                                          budget=wl.budget, k=wl.k, want_picked=True)
    idx, val, picked = idx.cpu().numpy(), val.cpu().numpy(), picked.cpu().numpy()
    P = d["centroids"].shape[0]
    _, _, det = bucket_select(d["q"], d["w"], d["centroids"], d["bucket_off"], d["bucket_mem"], d["keys"],
                              wl.top_p, wl.budget, wl.k, rows=rows, return_detail=True)
    keys = bf16_to_f64(d["keys"])
    recalls = []
    for i, t in enumerate(rows):
        cs = det[i]["centroid_scores"]
        check_set(picked[t], np.arange(P), cs, wl.top_p, RTOL_BF16, f"{name} picked row {t}")
        # expansion follows the GPU's pick order
        cand = expand_buckets(picked[t], d["bucket_off"], d["bucket_mem"], wl.budget)
        exact = indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], keys[cand])[0]
        check_selection(idx[t], val[t], cand, exact, wl.k, RTOL_BF16, f"{name} final row {t}")
        full = indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], keys)[0]
        ei, _ = select_topk(full, np.arange(keys.shape[0]), wl.k)
        recalls.append(recall_at_k(idx[t][None], ei[None]))
    return recalls


def test_bucket_small(L):
    rec = _check_bucket(L, "bucket_s", list(range(19)))
    assert min(rec) > 0.1


@pytest.mark.slow
def test_bucket_full_size_sampled(L):
    rec = _check_bucket(L, "bucket", [0, 100, 255])
    assert min(rec) > 0.3


# --------------------------------------------------------------------------- #
# native LSA flat search
# --------------------------------------------------------------------------- #
def _lsa_run(L, d, wl, threshold, fallback_rows=0):
    ex = wl.extra
    keys, n, picked = L.ls_lsa_flat_select(dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]),
                                           dev(d["bucket_off"]), dev(d["bucket_mem"]), block_keys=ex["block_keys"],
                                           buckets_per_block=ex["bpb"], n_sink=ex["n_sink"], top_p=wl.top_p,
                                           budget=wl.budget, threshold=threshold, fallback_rows=fallback_rows,
                                           want_picked=True)
    return keys.cpu().numpy(), n.cpu().numpy(), picked.cpu().numpy()


def _check_lsa(L, name, rows, d=None, wl=None, fallback_rows=0, compare_full=True):
    wl = wl or get_workload(name)
    d = d or data(name)
    ex = wl.extra
    keys, n, picked = _lsa_run(L, d, wl, threshold=True, fallback_rows=fallback_rows)
    if compare_full:
        # the full-matrix form picks the same buckets, bit for bit
        keys0, n0, picked0 = _lsa_run(L, d, wl, threshold=False)
        assert np.array_equal(picked0, picked) and np.array_equal(keys0, keys) and np.array_equal(n0, n), name
    _, det = lsa_flat_select(d["q_idx"], d["q_pos"], d["centroids"], d["bucket_off"], d["bucket_mem"],
                             ex["block_keys"], ex["bpb"], ex["n_sink"], wl.top_p, wl.budget, rows=rows,
                             return_detail=True)
    for i, t in enumerate(rows):
        v = det[i]["visible"]
        sc = det[i]["scores"]
        check_set(picked[t], np.arange(v), sc, wl.top_p, RTOL_BF16, f"{name} picked row {t}")
        got = picked[t][picked[t] >= 0]
        # best first by the reference scores, up to the tolerance
        gs = sc[got]
        assert np.all(gs[:-1] >= gs[1:] - RTOL_BF16 * max(1e-3, float(np.abs(sc).max(initial=0)))), t
        want = lsa_read_list(picked[t], d["q_pos"][t], d["bucket_off"], d["bucket_mem"], ex["block_keys"],
                             ex["n_sink"], wl.budget)
        assert n[t] == want.size and np.array_equal(keys[t, :n[t]], want), f"{name} read list row {t}"
        assert np.all(keys[t, n[t]:] == -1)


def test_lsa_flat_small(L):
    _check_lsa(L, "lsa_flat_s", list(range(37)))


@pytest.mark.slow
def test_lsa_flat_full_size_sampled(L):
    _check_lsa(L, "lsa_flat", [0, 1, 100, 254, 255])


def _missing_threshold_cases(base, top_p):
    """Every query points along u.  First: the sampled buckets (every
    top_p/16-th) point along u and the rest along -u, so the sample's 32nd
    best clears only sampled buckets: rows with fewer than top_p of them come
    up short.  Then all centroids along u, so every visible bucket ties at the
    threshold and rows with more than 4*top_p visible buckets overflow their
    lists."""
    from workloads.synth import to_bf16_bits
    rng = np.random.default_rng(3)
    u = rng.standard_normal(64)
    u /= np.linalg.norm(u)
    P = base["centroids"].shape[0]
    stride = max(1, top_p // 16)
    sign = np.where(np.arange(P) % stride == 0, 1.0, -1.0)
    for cent in (sign[:, None] * u[None, :], np.broadcast_to(u, (P, 64)).copy()):
        d = dict(base)
        d["q_idx"] = to_bf16_bits(np.broadcast_to(u, base["q_idx"].shape).copy())
        d["centroids"] = to_bf16_bits(cent)
        yield d


@pytest.mark.parametrize("fallback_rows", [0, 5])
def test_lsa_threshold_fallbacks(L, fallback_rows):
    """Rows whose sampled threshold misses fall back to full scoring, in one
    chunk of rows or in eight."""
    wl = get_workload("lsa_flat_s")
    for d in _missing_threshold_cases(data("lsa_flat_s"), wl.top_p):
        _check_lsa(L, "lsa_flat_s", list(range(37)), d=d, wl=wl, fallback_rows=fallback_rows)


def test_lsa_prefill_chunk_small(L):
    """A prefill chunk of 3000 queries: thirteen 256-query groups, each scored
    by a few of the scan's CTAs, so every row's list is shared among a few
    segments (proportional to the tiles each CTA scores)."""
    _check_lsa(L, "lsa_prefill_s", [0, 1, 255, 256, 1000, 2047, 2048, 2999])


def test_lsa_prefill_chunk_largest_top_p(L):
    """The 3000-query chunk with the largest top_p (4096): samples every
    256th bucket, lists of up to 16384, the 4096-entry top-k form."""
    from dataclasses import replace
    wl = replace(get_workload("lsa_prefill_s"), top_p=4096, budget=4096)
    _check_lsa(L, "lsa_prefill_s", [0, 1, 1000, 2999], wl=wl)


@pytest.mark.parametrize("fallback_rows", [0, 256, 700])
def test_lsa_prefill_chunk_fallbacks(L, fallback_rows):
    """Every row of the 3000-query chunk misses its threshold and is scored in
    full, 3000, 256 (12 chunks, the last ragged) or 700 rows at a time."""
    wl = get_workload("lsa_prefill_s")
    rows = [0, 1, 255, 256, 1000, 2999]
    for d in _missing_threshold_cases(data("lsa_prefill_s"), wl.top_p):
        _check_lsa(L, "lsa_prefill_s", rows, d=d, wl=wl, fallback_rows=fallback_rows)


@pytest.mark.slow
def test_lsa_prefill_10m_sampled(L):
    """The 32768-query chunk at 10M tokens: the threshold form only (the full
    matrix would take 172 GB), sampled rows against the oracle."""
    _check_lsa(L, "lsa_prefill_10m", [0, 1, 255, 256, 16383, 32767], compare_full=False)


def _check_lsa_tree(L, name, rows, beam=None):
    wl = get_workload(name)
    d = data(name)
    ex = wl.extra
    beam = beam or ex["beam"]
    fan, nblk = ex["fanout"], ex["node_block"]
    keys, n, picked, bm = L.ls_lsa_tree_select(
        dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]), dev_bf16(d["node_centroids"]),
        dev(d["bucket_off"]), dev(d["bucket_mem"]), block_keys=ex["block_keys"], buckets_per_block=ex["bpb"],
        node_block=nblk, fanout=fan, beam=beam, n_sink=ex["n_sink"], top_p=wl.top_p, budget=wl.budget,
        want_picked=True)
    keys, n, picked, bm = keys.cpu().numpy(), n.cpu().numpy(), picked.cpu().numpy(), bm.cpu().numpy()
    _, det = lsa_tree_select(d["q_idx"], d["q_pos"], d["centroids"], d["node_centroids"], d["bucket_off"],
                             d["bucket_mem"], ex["block_keys"], ex["bpb"], nblk, fan, beam, ex["n_sink"], wl.top_p,
                             wl.budget, rows=rows, return_detail=True)
    cent = bf16_to_f64(d["centroids"])
    for i, t in enumerate(rows):
        vn, v = det[i]["visible_nodes"], det[i]["visible"]
        check_set(bm[t], np.arange(vn), det[i]["node_scores"], beam, RTOL_BF16, f"{name} beam row {t}")
        # candidates from the GPU's beam: its children, then the uncovered buckets
        kept = bm[t][bm[t] >= 0]
        cand = np.asarray([int(x) * fan + c for x in kept for c in range(fan)] + list(range(vn * fan, v)),
                          dtype=np.int64)
        ref = cent[cand] @ bf16_to_f64(d["q_idx"][t]) if cand.size else np.zeros(0)
        check_set(picked[t], cand, ref, wl.top_p, RTOL_BF16, f"{name} picked row {t}")
        want = lsa_read_list(picked[t], d["q_pos"][t], d["bucket_off"], d["bucket_mem"], ex["block_keys"],
                             ex["n_sink"], wl.budget)
        assert n[t] == want.size and np.array_equal(keys[t, :n[t]], want), f"{name} read list row {t}"
        assert np.all(keys[t, n[t]:] == -1)


def test_lsa_tree_small(L):
    _check_lsa_tree(L, "lsa_flat_s", list(range(37)))


def test_lsa_tree_full_beam_matches_flat(L):
    """A beam covering every node bucket reads what the flat search reads
    (band rule on the picks: the two paths score on different units)."""
    _check_lsa_tree(L, "lsa_flat_s", list(range(37)), beam=4096)


@pytest.mark.slow
def test_lsa_tree_full_size_sampled(L):
    _check_lsa_tree(L, "lsa_tree", [0, 1, 100, 254, 255])


def _check_lsa_tree_levels(L, name, rows, beam=None, start_nodes=None, d=None):
    """Level by level against the oracle's scores of the candidates the GPU's
    own beam of the level above gives (band rule on each beam and on the
    picks), then the read lists exactly."""
    wl = get_workload(name)
    d = d or data(name)
    ex = wl.extra
    beam = beam or ex["beam"]
    start_nodes = start_nodes or ex["start_nodes"]
    fan, nblk = ex["fanout"], ex["node_block"]
    levels = d["node_levels"]
    keys, n, picked, bms = L.ls_lsa_tree_levels_select(
        dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]), [dev_bf16(x) for x in levels],
        dev(d["bucket_off"]), dev(d["bucket_mem"]), block_keys=ex["block_keys"], buckets_per_block=ex["bpb"],
        node_block=nblk, fanout=fan, beam=beam, start_nodes=start_nodes, n_sink=ex["n_sink"], top_p=wl.top_p,
        budget=wl.budget, want_picked=True)
    keys, n, picked, bms = keys.cpu().numpy(), n.cpu().numpy(), picked.cpu().numpy(), bms.cpu().numpy()
    _, det = lsa_tree_levels_select(d["q_idx"], d["q_pos"], d["centroids"], levels, d["bucket_off"],
                                    d["bucket_mem"], ex["block_keys"], ex["bpb"], nblk, fan, beam, start_nodes,
                                    ex["n_sink"], wl.top_p, wl.budget, rows=rows, return_detail=True)
    bits = [d["centroids"]] + list(levels)
    S = det[0]["start"]
    assert np.all(bms[S:] == -2), "levels above the start level are written"
    for i, t in enumerate(rows):
        v = det[i]["visible"]
        q = bf16_to_f64(d["q_idx"][t])
        cand = np.arange(v[S], dtype=np.int64)
        for lv in range(S, -1, -1):
            if lv < S:
                kept = bms[lv][t][bms[lv][t] >= 0]
                cand = np.asarray([int(x) * fan + c for x in kept for c in range(fan)]
                                  + list(range(fan * v[lv + 1], v[lv])), dtype=np.int64)
            ref = bf16_to_f64(bits[lv][cand]) @ q if cand.size else np.zeros(0)
            got = bms[lv - 1][t] if lv > 0 else picked[t]
            check_set(got, cand, ref, beam if lv > 0 else wl.top_p, RTOL_BF16, f"{name} level {lv} row {t}")
        want = lsa_read_list(picked[t], d["q_pos"][t], d["bucket_off"], d["bucket_mem"], ex["block_keys"],
                             ex["n_sink"], wl.budget)
        assert n[t] == want.size and np.array_equal(keys[t, :n[t]], want), f"{name} read list row {t}"
        assert np.all(keys[t, n[t]:] == -1)
    return keys, n, picked


@pytest.mark.parametrize("start_nodes", [100, 500, 5000])
def test_lsa_tree_levels_small(L, start_nodes):
    _check_lsa_tree_levels(L, "lsa_tree_levels_s", list(range(37)), start_nodes=start_nodes)


@pytest.mark.parametrize("beam", [1248, 4096])
def test_lsa_tree_levels_full_beam_matches_flat(L, beam):
    """A beam holding every visible entry of each level (1248, or the
    largest beam, 4096) reads what the flat search reads (band rule on the
    picks; read lists exactly)."""
    wl = get_workload("lsa_tree_levels_s")
    keys, n, picked = _check_lsa_tree_levels(L, "lsa_tree_levels_s", list(range(37)), beam=beam, start_nodes=100)
    _check_lsa(L, "lsa_tree_levels_s", list(range(37)), wl=wl)


def test_lsa_tree_levels_one_level_matches_one_level_search(L):
    """One node level: the same picks and read lists as the one-level search, bit for bit."""
    wl = get_workload("lsa_flat_s")
    d = data("lsa_flat_s")
    ex = wl.extra
    args = (dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]))
    kw = dict(block_keys=ex["block_keys"], buckets_per_block=ex["bpb"], node_block=ex["node_block"],
              fanout=ex["fanout"], beam=ex["beam"], n_sink=ex["n_sink"], top_p=wl.top_p, budget=wl.budget,
              want_picked=True)
    k1, n1, p1, _ = L.ls_lsa_tree_select(*args, dev_bf16(d["node_centroids"]), dev(d["bucket_off"]),
                                         dev(d["bucket_mem"]), **kw)
    k2, n2, p2, _ = L.ls_lsa_tree_levels_select(*args, [dev_bf16(d["node_centroids"])], dev(d["bucket_off"]),
                                                dev(d["bucket_mem"]), start_nodes=32768, **kw)
    assert torch.equal(p1, p2) and torch.equal(k1, k2) and torch.equal(n1, n2)


def test_lsa_tree_levels_empty_start_level(L):
    """The start level holds no node (level sizes 1024 and 0, start_nodes 1):
    an empty beam, every level-1 node uncovered, then the buckets."""
    from workloads.synth import make_lsa
    d = make_lsa(37, 40000, 512, 64, 0, 2053, True, node_block=4096, fanout=4, levels=2)
    assert [x.shape[0] for x in d["node_levels"]] == [1024, 0]
    _check_lsa_tree_levels(L, "lsa_flat_s", list(range(37)), beam=96, start_nodes=1, d=d)


@pytest.mark.slow
def test_lsa_tree_levels_10m_sampled(L):
    _check_lsa_tree_levels(L, "lsa_tree_10m", [0, 1, 100, 254, 255])


def test_bucket_bad_member_flagged(L):
    d = data("bucket_s")
    mem = d["bucket_mem"].copy()
    mem[:] = np.where(np.arange(mem.size) % 5 == 0, d["keys"].shape[0] + 1000, mem)  # out of range ids
    L.ls_device_status()
    L.ls_bucket_select(dev_bf16(d["q"]), dev(d["w"]), dev_bf16(d["centroids"]), dev(d["bucket_off"]), dev(mem),
                       dev_bf16(d["keys"]), top_p=64, budget=512, k=512)
    flags = L.ls_device_status()
    assert flags & 2  # LS_FAULT_BAD_INDEX: the bad rows were skipped, not read


# --------------------------------------------------------------------------- #
# failure detection: a bounded device wait ends with an error status
# --------------------------------------------------------------------------- #
def test_wait_probe_times_out_and_context_survives(L):
    L.ls_device_status()
    gave_up = L.ls_selftest_wait_probe(2_000_000)  # 2 ms
    flags = L.ls_device_status()
    assert int(gave_up.item()) == 1
    assert flags & 1
    # the context is still usable
    test_decode_edge_rows(L)


# --------------------------------------------------------------------------- #
# the selection histogram the scans count for the top-k
# --------------------------------------------------------------------------- #
def _order_codes(x):
    """Order-preserving codes of fp32 scores, restated here for the check:
    NaN -> 0, -0.0 -> code of +0.0, negatives bit-inverted, positives with the
    sign bit set."""
    x = np.asarray(x, np.float32)
    b = x.view(np.uint32).copy()
    b[b == 0x80000000] = 0
    code = np.where(b & 0x80000000, ~b, b | 0x80000000).astype(np.uint32)
    code[np.isnan(x)] = 0
    return code


@pytest.mark.parametrize("fmt", ["bf16", "int8"])
def test_scan_histogram_feeds_topk(L, fmt):
    name = "decode_s" if fmt == "bf16" else "two_stage_s"
    d = data(name)
    B, H, dd = d["q"].shape
    q, w, nv = dev_bf16(d["q"]), dev(d["w"]), dev(d["n_valid"])
    hist = torch.zeros((B, 2048), dtype=torch.int32, device="cuda")
    if fmt == "bf16":
        sc = L.ls_indexer_score(q.view(B, 1, H, dd), w.view(B, 1, H), dev_bf16(d["k"]), n_valid=nv, hist_out=hist)
    else:
        sc = L.ls_indexer_score(q.view(B, 1, H, dd), w.view(B, 1, H), dev(d["ck"]), key_scale=dev(d["ck_scale"]),
                                n_valid=nv, hist_out=hist)
    sc = sc[:, 0].contiguous()
    s_np = sc.cpu().numpy()
    h_np = hist.cpu().numpy()
    for b in range(B):
        n = int(d["n_valid"][b])
        ref = np.bincount(_order_codes(s_np[b, :n]) >> 21, minlength=2048)
        assert np.array_equal(h_np[b], ref), f"histogram row {b}"
    for k in (1, 512, 1024):
        i1, v1 = L.ls_topk_select(sc, k, n_valid=nv, hist=hist)
        i0, v0 = L.ls_topk_select(sc, k, n_valid=nv)
        ri, rv = topk_rows(s_np, d["n_valid"], k)
        assert np.array_equal(i1.cpu().numpy(), ri) and f32_bits_equal(v1.cpu().numpy(), rv)
        assert np.array_equal(i0.cpu().numpy(), ri) and f32_bits_equal(v0.cpu().numpy(), rv)


def test_profiling_counts_launches(L):
    d = data("decode_tiny")
    q, w, k = dev_bf16(d["q"]), dev(d["w"]), dev_bf16(d["k"])
    L.ls_profile_begin()
    for _ in range(3):
        L.ls_decode_select(q, w, k, 512)
    prof = L.ls_profile_end()
    assert prof["score_tc_kernel<1>"][1] == 3 and prof["topk_kernel"][1] == 3
    assert all(ms > 0 for ms, _ in prof.values())
