"""Pins of the fp64 oracle against facts fixed outside it (no GPU).

Each test checks the oracle against something it cannot simply repeat: the
formats' library decoders, pure-Python brute force, closed forms, invariants,
explicit block construction, the pages' printed figures.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute, sizes
from oracle.formats import bf16_to_f64, dequant, e4m3_to_f64, f16_to_f64, int8_to_f64, pq_decode
from oracle.indexer import eligible_blocks, eligible_count, indexer_scores
from oracle.select import (
    bucket_select, decode_select, expand_buckets, lsa_flat_select, lsa_read_list, lsa_tree_levels,
    lsa_tree_levels_select,
    lsa_tree_select, lsa_visible, prefill_select,
    prefill_select_fp8, recall_at_k, select_topk, topk_rows, two_stage_pq_select, two_stage_select,
)
from workloads import get_workload, make_workload
from workloads.synth import make_bucket, make_decode, make_two_stage, to_bf16_bits


# --------------------------------------------------------------------------- #
# formats: every code against the library casts
# --------------------------------------------------------------------------- #
def test_bf16_decode_all_codes():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    with np.errstate(invalid="ignore"):        # widening the signalling-NaN codes raises the invalid flag
        got = bf16_to_f64(bits)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(got[~both_nan], ref[~both_nan])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_to_f64(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    # a few fixed points of the format: max finite, smallest subnormal, 1.0
    assert e4m3_to_f64(np.array([0x7E]))[0] == 448.0
    assert e4m3_to_f64(np.array([0x01]))[0] == 2.0 ** -9
    assert e4m3_to_f64(np.array([0x38]))[0] == 1.0
    assert e4m3_to_f64(np.array([0xB8]))[0] == -1.0


def test_int8_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.int8).to(torch.float64).numpy()
    assert np.array_equal(int8_to_f64(codes), ref)
    assert int8_to_f64(np.array([0x80], np.uint8))[0] == -128.0 and int8_to_f64(np.array([0x7F], np.uint8))[0] == 127.0


def test_f16_decode_all_codes():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = f16_to_f64(bits)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert f16_to_f64(np.array([0x7BFF]))[0] == 65504.0
    assert f16_to_f64(np.array([0x0001]))[0] == 2.0 ** -24
    assert f16_to_f64(np.array([0x3C00]))[0] == 1.0
    assert f16_to_f64(np.array([0xFC00]))[0] == -np.inf


def test_pq_decode_brute_force():
    rng = np.random.default_rng(21)
    books = (rng.standard_normal((32, 256, 4)) * 0.1).astype(np.float16).view(np.uint16)
    codes = rng.integers(0, 256, size=(5, 32)).astype(np.uint8)
    got = pq_decode(codes, books)
    for r in range(5):
        want = []
        for m in range(32):
            for j in range(4):
                want.append(float(np.float16(books[m, codes[r, m], j].view(np.float16))))
        assert got[r].tolist() == want


def test_pq_generator_codes_are_nearest_centroids():
    d = make_two_stage(B=2, N=900, seed=22, plant_frac=0.05, ragged=200, pq=True, pq_sample=1200)
    books = f16_to_f64(d["pq_books"])                                  # [32, 256, 4]
    keys = dequant(d["fk"][1, :50], d["fk_scale"][1, :50], "e4m3")      # [50, 128]
    for m in range(32):
        x = keys[:, 4 * m: 4 * m + 4]
        d2 = ((x[:, None, :] - books[m][None]) ** 2).sum(-1)            # [50, 256]
        chosen = d2[np.arange(50), d["pq_codes"][1, :50, m].astype(np.int64)]
        assert np.all(chosen <= d2.min(1) * (1 + 1e-5) + 1e-12)


def test_two_stage_pq_full_shortlist_equals_exact():
    d = make_two_stage(B=2, N=700, seed=23, plant_frac=0.05, ragged=100, pq=True, pq_sample=1000)
    n = d["n_valid"]
    got_i, got_v = two_stage_pq_select(d["q"], d["w"], d["pq_codes"], d["pq_books"], d["fk"], d["fk_scale"], n,
                                       shortlist=700, k=32)
    for b in range(2):
        keys = dequant(d["fk"][b, : n[b]], d["fk_scale"][b, : n[b]], "e4m3")
        s = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None], keys)[0]
        ei, ev = select_topk(s, np.arange(n[b]), 32)
        assert np.array_equal(got_i[b], ei)
        assert np.array_equal(got_v[b], ev)


def test_two_stage_pq_brute_force_tiny():
    d = make_two_stage(B=1, N=60, seed=24, plant_frac=0.1, pq=True, pq_sample=60)
    gi, gv, det = two_stage_pq_select(d["q"], d["w"], d["pq_codes"], d["pq_books"], d["fk"], d["fk_scale"],
                                      d["n_valid"], shortlist=12, k=5, return_detail=True)
    qb = bf16_to_f64(d["q"][0]).tolist()
    wb = d["w"][0].astype(np.float64).tolist()
    books = d["pq_books"].view(np.float16)
    ck = [[float(books[m, d["pq_codes"][0, s, m], j]) for m in range(32) for j in range(4)] for s in range(60)]
    fk = e4m3_to_f64(d["fk"][0]) * d["fk_scale"][0].astype(np.float64)[:, None]
    shat = [brute.score(qb, wb, ck[s]) for s in range(60)]
    short, _ = brute.topk(shat, list(range(60)), 12)
    ex = [brute.score(qb, wb, fk[s].tolist()) for s in short]
    bp, _ = brute.topk(ex, short, 5)
    assert gi[0].tolist() == bp
    assert det[0]["shortlist"].tolist() == short


def test_dequant_scales():
    codes = np.array([[0x38, 0x40]], dtype=np.uint8)  # 1.0, 2.0
    v = dequant(codes, np.array([0.5], np.float32), "e4m3")
    assert np.array_equal(v, [[0.5, 1.0]])
    v = dequant(np.array([[-127, 3]], np.int8), np.array([0.25], np.float32), "int8")
    assert np.array_equal(v, [[-31.75, 0.75]])


# --------------------------------------------------------------------------- #
# scores
# --------------------------------------------------------------------------- #
def test_scores_closed_form():
    # H=2, d=2.  Head 0 sees +k0 dims, head 1 sees -k0: exactly one ReLU is open.
    q = np.array([[[1.0, 0.0], [-1.0, 0.0]]])
    w = np.array([[2.0, -3.0]])
    k = np.array([[5.0, 7.0], [-2.0, 11.0]])
    s = indexer_scores(q, w, k)
    # s0 = 2*max(0,5) - 3*max(0,-5) = 10 ; s1 = 2*max(0,-2) - 3*max(0,2) = -6
    assert np.array_equal(s, [[10.0, -6.0]])


def test_scores_brute_force_tiny():
    rng = np.random.default_rng(1)
    T, H, d, N = 3, 4, 5, 9
    q = rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H))
    k = rng.standard_normal((N, d))
    got = indexer_scores(q, w, k)
    for t in range(T):
        for s in range(N):
            ref = brute.score(q[t].tolist(), w[t].tolist(), k[s].tolist())
            assert abs(got[t, s] - ref) <= 1e-12 * (1 + abs(ref))


def test_scores_gemv_special_case():
    # one head, unit weight, every dot positive: the score is a plain GEMV
    rng = np.random.default_rng(2)
    q = np.abs(rng.standard_normal((1, 1, 16)))
    k = np.abs(rng.standard_normal((33, 16)))
    got = indexer_scores(q, np.ones((1, 1)), k)[0]
    assert np.allclose(got, np.dot(k, q[0, 0]), rtol=1e-14, atol=0)


def test_scores_invariants():
    rng = np.random.default_rng(3)
    T, H, d, N = 2, 6, 8, 20
    q = rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H))
    k = rng.standard_normal((N, d))
    s = indexer_scores(q, w, k)
    # positive homogeneity of ReLU in q and linearity in w
    assert np.allclose(indexer_scores(2.5 * q, w, k), 2.5 * s, rtol=1e-12, atol=1e-12)
    assert np.allclose(indexer_scores(q, -w, k), -s, rtol=1e-12, atol=1e-12)
    # heads are a set: permuting them together with w changes nothing
    perm = rng.permutation(H)
    assert np.allclose(indexer_scores(q[:, perm], w[:, perm], k), s, rtol=1e-12, atol=1e-12)
    # keys are positions: permuting keys permutes the scores
    kp = rng.permutation(N)
    assert np.allclose(indexer_scores(q, w, k[kp]), s[:, kp], rtol=1e-12, atol=1e-12)
    # a head whose dots are all negative contributes nothing
    q2 = q.copy()
    q2[:, 0] = 0.0
    w2 = w.copy()
    w2[:, 0] = 1e6
    assert np.allclose(indexer_scores(q2, w2, k), indexer_scores(q2[:, 1:], w2[:, 1:], k))


# --------------------------------------------------------------------------- #
# eligibility
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("stride", [1, 2, 3, 4])
def test_eligibility_matches_blocks(stride):
    n_keys = 12
    for t in range(0, 4 * n_keys + 3):
        blocks = eligible_blocks(t, stride, n_keys)
        n = int(eligible_count(np.array([t]), stride, n_keys)[0])
        assert blocks == list(range(n)), (t, stride)


def test_eligibility_edges_stride4():
    # t = 0..7: the first block [0..3] completes at t = 3, the second at t = 7
    got = eligible_count(np.arange(8), 4, 100).tolist()
    assert got == [0, 0, 0, 1, 1, 1, 1, 2]


def test_prefill_chunk_eligible_pairs():
    t = np.arange(126976, 131072)
    n = eligible_count(t, 4, 32768)
    assert n.min() == 31744 and n.max() == 32768
    assert int(n.sum()) == 132119552


# --------------------------------------------------------------------------- #
# top-k order
# --------------------------------------------------------------------------- #
def _check_topk_vs_brute(vals, k):
    pos = list(range(len(vals)))
    bp, bv = brute.topk([float(v) for v in vals], pos, k)
    gp, gv = select_topk(np.asarray(vals), np.arange(len(vals)), k)
    assert gp.tolist() == bp
    for a, b in zip(gv.tolist(), bv):
        assert (math.isnan(a) and math.isnan(b)) or a == b


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(4)
    for trial in range(30):
        n = int(rng.integers(1, 60))
        vals = rng.integers(-3, 4, size=n).astype(np.float64)
        if trial % 3 == 0:
            vals[rng.integers(0, n, size=max(1, n // 5))] = np.nan
        if trial % 4 == 0:
            vals[rng.integers(0, n, size=max(1, n // 5))] = -np.inf
        for k in (1, 5, n, n + 3):
            _check_topk_vs_brute(vals, k)


def test_topk_adversarial():
    # all equal: the first k positions
    p, _ = select_topk(np.zeros(100, np.float32), np.arange(100), 10)
    assert p.tolist() == list(range(10))
    # -0.0 ties +0.0: lower position first whatever the sign bit
    v = np.array([0.0, -0.0, 0.0, -0.0], np.float32)
    p, val = select_topk(v, np.arange(4), 4)
    assert p.tolist() == [0, 1, 2, 3]
    assert np.signbit(val).tolist() == [False, True, False, True]
    # -inf above NaN, NaN above padding
    v = np.array([np.nan, -np.inf, 1.0], np.float32)
    p, val = select_topk(v, np.arange(3), 5)
    assert p.tolist() == [2, 1, 0, -1, -1]
    assert val[3] == -np.inf and math.isnan(val[2])
    # duplicated maxima
    v = np.array([1, 5, 5, 2, 5], np.float32)
    p, _ = select_topk(v, np.arange(5), 2)
    assert p.tolist() == [1, 2]
    # positions are labels, not indexes: ties go to the lower label
    p, _ = select_topk(np.array([1.0, 1.0]), np.array([9, 4]), 1)
    assert p.tolist() == [4]


def test_topk_rows_prefix_and_padding():
    s = np.array([[3, 1, 2, 9], [5, 5, 5, 5]], np.float32)
    idx, val = topk_rows(s, np.array([3, 0]), 2)
    assert idx.tolist() == [[0, 2], [-1, -1]]
    assert val.dtype == np.float32


def test_topk_is_prefix_of_full_sort():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(500).astype(np.float32)
    v[::7] = v[3]
    full_p, _ = brute.full_sort(v.tolist(), list(range(500)))
    for k in (1, 17, 128, 499):
        p, _ = select_topk(v, np.arange(500), k)
        assert p.tolist() == full_p[:k]


# --------------------------------------------------------------------------- #
# pipelines
# --------------------------------------------------------------------------- #
def test_decode_select_brute_force_tiny():
    data = make_decode(B=2, N=40, H=3, d=6, seed=7, n_valid=np.array([40, 23]))
    idx, val = decode_select(data["q"], data["w"], data["k"], data["n_valid"], k=8)
    for b in range(2):
        n = int(data["n_valid"][b])
        qb = bf16_to_f64(data["q"][b]).tolist()
        kb = bf16_to_f64(data["k"][b, :n]).tolist()
        sc = [brute.score(qb, data["w"][b].astype(np.float64).tolist(), kb[s]) for s in range(n)]
        bp, bv = brute.topk(sc, list(range(n)), 8)
        assert idx[b].tolist() == bp
        assert np.allclose(val[b], bv, rtol=1e-12, atol=1e-15)


def test_prefill_select_brute_force_tiny():
    data = make_workload("prefill_s")
    q, w, k, q_pos = data["q"][:4, :3, :], data["w"][:4, :3], data["k"][:80], data["q_pos"][:4] - 3800
    idx, val = prefill_select(q, w, q_pos, k, stride=4, k=16)
    kf = bf16_to_f64(k).tolist()
    for t in range(4):
        elig = eligible_blocks(int(q_pos[t]), 4, 80)
        sc = [brute.score(bf16_to_f64(q[t]).tolist(), w[t].astype(np.float64).tolist(), kf[s]) for s in elig]
        bp, bv = brute.topk(sc, elig, 16)
        assert idx[t].tolist() == bp


def _e4m3_code_of_int(v: int) -> int:
    """The e4m3 code of an integer |v| <= 15, built from the field layout
    (sign, exponent biased by 7, 3 mantissa bits)."""
    v = int(v)
    s = 0x80 if v < 0 else 0
    a = abs(v)
    if a == 0:
        return s
    e = a.bit_length() - 1
    m = ((a - (1 << e)) * 8) >> e
    return s | ((e + 7) << 3) | m


def test_prefill_select_fp8_integer_codes_brute_force():
    """fp8 codes of small integers with power-of-two scales: every product and
    sum is exact in fp64, so the oracle's scores equal a pure-Python brute
    force exactly; a scale applied to the wrong axis changes them."""
    rng = np.random.default_rng(11)
    T, H, d, N = 5, 3, 8, 40
    qi = rng.integers(-15, 16, size=(T, H, d))
    ki = rng.integers(-15, 16, size=(N, d))
    q8 = np.vectorize(_e4m3_code_of_int)(qi).astype(np.uint8)
    k8 = np.vectorize(_e4m3_code_of_int)(ki).astype(np.uint8)
    assert np.array_equal(e4m3_to_f64(q8), qi) and np.array_equal(e4m3_to_f64(k8), ki)
    qs = np.exp2(rng.integers(-3, 4, size=(T, H))).astype(np.float32)
    ks = np.exp2(rng.integers(-3, 4, size=N)).astype(np.float32)
    w = rng.standard_normal((T, H)).astype(np.float32)
    q_pos = np.array([3, 40, 99, 150, 159], dtype=np.int64)
    idx, val, scores = prefill_select_fp8(q8, qs, w, q_pos, k8, ks, stride=4, k=8, return_scores=True)
    for t in range(T):
        n = min((int(q_pos[t]) + 1) // 4, N)
        qt = [[float(qi[t, h, j]) * float(qs[t, h]) for j in range(d)] for h in range(H)]
        ref = [brute.score(qt, [float(x) for x in w[t]], [float(ki[s, j]) * float(ks[s]) for j in range(d)])
               for s in range(n)]
        assert scores[t].tolist() == ref
        bp, _ = brute.topk(ref, list(range(n)), 8)
        assert idx[t].tolist() == bp


def test_prefill_select_fp8_equals_bf16_pipeline():
    """Every e4m3 value times a power of two is a bf16 value: the fp8
    selection must equal the bf16 selection of the decoded inputs."""
    d = make_workload("prefill_fp8_s")
    rows = np.array([0, 5, 40, 76])
    qs = np.exp2(np.round(np.log2(d["q_scale"]))).astype(np.float32)
    ks = np.exp2(np.round(np.log2(d["k_scale"]))).astype(np.float32)
    qb = to_bf16_bits(e4m3_to_f64(d["q8"]) * qs[..., None])
    kb = to_bf16_bits(e4m3_to_f64(d["k8"]) * ks[:, None])
    assert np.array_equal(bf16_to_f64(qb), e4m3_to_f64(d["q8"]) * qs[..., None].astype(np.float64))
    i8, v8 = prefill_select_fp8(d["q8"], qs, d["w"], d["q_pos"], d["k8"], ks, stride=4, k=64, rows=rows)
    ib, vb = prefill_select(qb, d["w"], d["q_pos"], kb, stride=4, k=64, rows=rows)
    assert np.array_equal(i8, ib) and np.array_equal(v8, vb)


def test_fp8_prefill_generator_scales():
    """The fp8 inputs are the bf16 draws quantised per row: scale = amax / 448
    and every decoded value within half an e4m3 step of the original."""
    d = make_workload("prefill_fp8_s")
    qf = bf16_to_f64(d["q"])
    amax = np.abs(qf).max(axis=-1)
    assert np.allclose(d["q_scale"], (amax / 448.0).astype(np.float32))
    deq = e4m3_to_f64(d["q8"]) * d["q_scale"].astype(np.float64)[..., None]
    assert np.all(np.abs(deq - qf) <= np.abs(qf) * 2.0 ** -4 + d["q_scale"][..., None] * 2.0 ** -9)


def test_lsa_visibility_by_blocks():
    """A bucket is visible iff its whole block ends at or before the start of
    the query's own block (brute force over blocks)."""
    block_keys, bpb, P = 16, 3, 3 * 7
    for t in range(0, 16 * 9):
        wstart = (t // block_keys) * block_keys
        vis = [p for p in range(P) if (p // bpb + 1) * block_keys <= wstart]
        assert lsa_visible([t], block_keys, bpb, P)[0] == len(vis)
        assert vis == list(range(len(vis)))


def test_lsa_dot_equals_two_head_indexer_score():
    """The single dot product is the indexer score with heads q and -q,
    weights 1 and -1: max(0, x) - max(0, -x) = x."""
    d = make_workload("lsa_flat_s")
    q = bf16_to_f64(d["q_idx"][:5])
    c = bf16_to_f64(d["centroids"][:300])
    qq = np.stack([q, -q], axis=1)                       # [5, 2, 64]
    w = np.tile(np.array([1.0, -1.0]), (5, 1))
    assert np.allclose(indexer_scores(qq, w, c), q @ c.T, rtol=0, atol=1e-15)
    _, det = lsa_flat_select(d["q_idx"], d["q_pos"], d["centroids"], d["bucket_off"], d["bucket_mem"], 512, 64, 4,
                             64, 512, rows=[11], return_detail=True)
    assert np.allclose(det[0]["scores"], indexer_scores(np.stack([bf16_to_f64(d["q_idx"][11]),
                                                                  -bf16_to_f64(d["q_idx"][11])])[None],
                                                        np.array([[1.0, -1.0]]), bf16_to_f64(d["centroids"]))[0],
                       rtol=0, atol=1e-15)


def test_lsa_read_list_covers_history_with_full_budget():
    """With every visible bucket picked and an unlimited budget, the read list
    is exactly the positions 0 .. t, each once."""
    d = make_workload("lsa_flat_s")
    for t in (0, 3, 4, 511, 512, 1024, 5000, 39999):
        qpos = d["q_pos"].copy()
        qpos[0] = t
        out = lsa_flat_select(d["q_idx"], qpos, d["centroids"], d["bucket_off"], d["bucket_mem"], 512, 64,
                              4, 4096, 10 ** 6, rows=[0])[0]
        if t // 512 * 64 <= 4096:
            assert sorted(out.tolist()) == list(range(t + 1)), t


def test_lsa_brute_force_tiny():
    """Pure-Python dot products and a full sort pick the buckets; the read
    list of the picked order is rebuilt by hand."""
    d = make_workload("lsa_flat_s")
    t = 5000
    v = (t // 512) * 64
    cent = bf16_to_f64(d["centroids"]).tolist()
    q = bf16_to_f64(d["q_idx"][20:21])[0].tolist()
    scores = [sum(a * b for a, b in zip(cent[p], q)) for p in range(v)]
    bp, _ = brute.topk(scores, list(range(v)), 16)
    qpos = d["q_pos"].copy()
    qpos[20] = t
    out, det = lsa_flat_select(d["q_idx"], qpos, d["centroids"], d["bucket_off"], d["bucket_mem"], 512, 64, 4, 16,
                               100, rows=[20], return_detail=True)
    assert det[0]["picked"].tolist() == bp
    want = [0, 1, 2, 3] + list(range(4608, 5001))
    for p in bp:
        for m in d["bucket_mem"][d["bucket_off"][p]:d["bucket_off"][p + 1]]:
            if 4 <= m < 4608 and len(want) < 4 + 393 + 100:
                want.append(int(m))
    assert out[0].tolist() == want
    assert lsa_read_list(bp, t, d["bucket_off"], d["bucket_mem"], 512, 4, 100).tolist() == want


def test_lsa_tree_with_full_beam_equals_flat():
    """A beam holding every visible node bucket steps down to every visible
    bucket: the tree search reads what the flat search reads."""
    d = make_workload("lsa_flat_s")
    args = (d["q_idx"], d["q_pos"], d["centroids"])
    flat = lsa_flat_select(*args, d["bucket_off"], d["bucket_mem"], 512, 64, 4, 64, 512)
    tree = lsa_tree_select(*args, d["node_centroids"], d["bucket_off"], d["bucket_mem"], 512, 64, 4096, 4, 4096,
                           4, 64, 512)
    for t in range(d["q_pos"].size):
        assert np.array_equal(flat[t], tree[t]), t


def test_lsa_tree_brute_force_tiny():
    """Pure-Python node scores, beam, children + uncovered buckets, picks."""
    d = make_workload("lsa_flat_s")
    t = int(np.argmax(d["q_pos"]))
    v = min((int(d["q_pos"][t]) // 512) * 64, d["centroids"].shape[0])
    vn = (v // 4096) * 1024
    assert vn > 0 and v > vn * 4
    q = bf16_to_f64(d["q_idx"][t:t + 1])[0].tolist()
    nodes = bf16_to_f64(d["node_centroids"]).tolist()
    cent = bf16_to_f64(d["centroids"]).tolist()
    ns = [sum(a * b for a, b in zip(nodes[n], q)) for n in range(vn)]
    beam, _ = brute.topk(ns, list(range(vn)), 7)
    cand = [4 * n + c for n in beam for c in range(4)] + list(range(vn * 4, v))
    cs = [sum(a * b for a, b in zip(cent[p], q)) for p in cand]
    picked, _ = brute.topk(cs, cand, 20)
    out, det = lsa_tree_select(d["q_idx"], d["q_pos"], d["centroids"], d["node_centroids"], d["bucket_off"],
                               d["bucket_mem"], 512, 64, 4096, 4, 7, 4, 20, 100, rows=[t], return_detail=True)
    assert det[0]["beam"].tolist() == beam
    assert det[0]["picked"].tolist() == picked
    assert out[0].tolist() == lsa_read_list(picked, d["q_pos"][t], d["bucket_off"], d["bucket_mem"], 512, 4,
                                            100).tolist()


def test_lsa_generator_node_centroids():
    """Node centroid = the normalised sum of its 4 children's key sums, each
    taken as size x centroid."""
    d = make_workload("lsa_flat_s")
    sizes = np.diff(d["bucket_off"]).astype(np.float64)
    c = bf16_to_f64(d["centroids"])
    n = bf16_to_f64(d["node_centroids"])
    for j in (0, 1, 511, 1023):
        s = (c[4 * j:4 * j + 4] * sizes[4 * j:4 * j + 4, None]).sum(axis=0)
        assert np.allclose(n[j], s / np.linalg.norm(s), atol=2 ** -8)


def _levels_args(d, ex):
    return (d["q_idx"], d["q_pos"], d["centroids"], d["node_levels"], d["bucket_off"], d["bucket_mem"],
            ex["block_keys"], ex["bpb"], ex["node_block"], ex["fanout"])


@pytest.mark.parametrize("start_nodes", [100, 500, 5000])
def test_lsa_tree_levels_with_full_beam_equals_flat(start_nodes):
    """A beam holding every visible entry of each level steps down to every
    visible bucket, from whichever level it starts: the tree reads what the
    flat search reads."""
    wl = get_workload("lsa_tree_levels_s")
    d = make_workload("lsa_tree_levels_s")
    ex = wl.extra
    flat = lsa_flat_select(d["q_idx"], d["q_pos"], d["centroids"], d["bucket_off"], d["bucket_mem"],
                           ex["block_keys"], ex["bpb"], ex["n_sink"], wl.top_p, wl.budget)
    tree, det = lsa_tree_levels_select(*_levels_args(d, ex), 5000, start_nodes, ex["n_sink"], wl.top_p, wl.budget,
                                       return_detail=True)
    assert det[0]["start"] == {100: 3, 500: 2, 5000: 1}[start_nodes]
    for t in range(d["q_pos"].size):
        assert np.array_equal(flat[t], tree[t]), t


def test_lsa_tree_levels_one_level_equals_one_level_search():
    """With one node level the search is the one-level tree search."""
    wl = get_workload("lsa_flat_s")
    d = make_workload("lsa_flat_s")
    ex = wl.extra
    args = (d["q_idx"], d["q_pos"], d["centroids"])
    one = lsa_tree_select(*args, d["node_centroids"], d["bucket_off"], d["bucket_mem"], 512, 64, 4096, 4, 96, 4,
                          64, 512)
    lv = lsa_tree_levels_select(*args, [d["node_centroids"]], d["bucket_off"], d["bucket_mem"], 512, 64, 4096, 4,
                                96, 32768, 4, 64, 512)
    for t in range(d["q_pos"].size):
        assert np.array_equal(one[t], lv[t]), t


@pytest.mark.parametrize("node_block,fanout", [(16, 4), (8, 2), (12, 3)])
def test_lsa_tree_levels_by_explicit_blocks(node_block, fanout):
    """Level l's node j exists for a query when every entry of its node
    cluster block at level l - 1 is visible: the block of node j is entries
    (j // (node_block / fanout)) * node_block ... + node_block - 1 below.
    Counted here entry by entry, up to each level's size."""
    per = node_block // fanout
    sizes = [97, 30, 9, 2]                               # level sizes 1..4 (level 0: the visible buckets)
    for vis in range(0, 400, 3):
        want, below = [vis], vis
        for size in sizes:
            n = sum(1 for j in range(size) if (j // per) * node_block + node_block <= below)
            want.append(n)
            below = n
        assert lsa_tree_levels(vis, sizes, node_block, fanout) == want, vis
    # 1M tokens: 131072 buckets in 32 complete 4096-bucket blocks -> 32768 level-1 nodes
    assert lsa_tree_levels(131072, [32768, 8192], 4096, 4) == [131072, 32768, 8192]
    assert lsa_tree_levels(131071, [32768, 8192], 4096, 4) == [131071, 31744, 7168]


@pytest.mark.parametrize("start_nodes,beam", [(100, 5), (500, 7), (5000, 9)])
def test_lsa_tree_levels_brute_force_tiny(start_nodes, beam):
    """Pure-Python levels: the visible entries of a level are those whose
    block of node_block entries below is complete and visible; an entry is
    covered when its parent is visible; the start level is scored in full,
    every level below over the beam's children and the uncovered entries."""
    wl = get_workload("lsa_tree_levels_s")
    d = make_workload("lsa_tree_levels_s")
    ex = wl.extra
    fan, blk = ex["fanout"], ex["node_block"]
    lv_bits = [d["centroids"]] + d["node_levels"]
    start = {100: 3, 500: 2, 5000: 1}[start_nodes]
    rows = [t for t in range(d["q_pos"].size) if d["q_pos"][t] >= 9000][:5] + [4, 8, 11, 0]
    out, det = lsa_tree_levels_select(*_levels_args(d, ex), beam, start_nodes, ex["n_sink"], wl.top_p, wl.budget,
                                      rows=rows, return_detail=True)
    for i, t in enumerate(rows):
        q = bf16_to_f64(d["q_idx"][t:t + 1])[0].tolist()
        vis = [min(int(d["q_pos"][t]) // 512 * 64, d["centroids"].shape[0])]
        for lv in range(1, 4):
            n_up = lv_bits[lv].shape[0]
            # node n exists for the query when all of its block's entries below are visible
            vis.append(sum(1 for n in range(n_up) if ((n * fan) // blk + 1) * blk <= vis[lv - 1]))
        kept = None
        for lv in range(start, -1, -1):
            if kept is None:
                cand = list(range(vis[lv]))
            else:
                cand = [c for c in range(vis[lv]) if c // fan in kept or c // fan >= vis[lv + 1]]
            rows_f = bf16_to_f64(lv_bits[lv][cand]).tolist() if cand else []
            sc = [sum(a * b for a, b in zip(r, q)) for r in rows_f]
            k = beam if lv > 0 else wl.top_p
            sel, _ = brute.topk(sc, cand, k)
            sel = [x for x in sel if x >= 0]
            if lv > 0:
                assert sorted(det[i]["beams"][lv].tolist()) == sorted(sel), (t, lv)
                kept = set(sel)
            else:
                assert [x for x in det[i]["picked"].tolist() if x >= 0] == sel, t
        want = lsa_read_list(np.asarray(sel + [-1] * (wl.top_p - len(sel))), d["q_pos"][t], d["bucket_off"],
                             d["bucket_mem"], 512, ex["n_sink"], wl.budget)
        assert out[i].tolist() == want.tolist(), t


def test_lsa_tree_levels_empty_start_level_equals_flat_with_full_beam():
    """A tree whose top level has no node (4992 buckets, node blocks of 4096:
    1024 level-1 nodes, none at level 2) started there: every level-1 node is
    uncovered and joins the level-1 candidates, so a full beam still reads
    what the flat search reads."""
    from workloads.synth import make_lsa
    d = make_lsa(37, 40000, 512, 64, 0, 2053, True, node_block=4096, fanout=4, levels=2)
    assert [x.shape[0] for x in d["node_levels"]] == [1024, 0]
    flat = lsa_flat_select(d["q_idx"], d["q_pos"], d["centroids"], d["bucket_off"], d["bucket_mem"], 512, 64, 4,
                           64, 512)
    tree, det = lsa_tree_levels_select(d["q_idx"], d["q_pos"], d["centroids"], d["node_levels"], d["bucket_off"],
                                       d["bucket_mem"], 512, 64, 4096, 4, 5000, 1, 4, 64, 512, return_detail=True)
    assert det[0]["start"] == 2
    for t in range(d["q_pos"].size):
        assert np.array_equal(flat[t], tree[t]), t


def test_lsa_tree_levels_counts_match_page_figures(golden_dir):
    """The beam rule replayed at 1M and 10M tokens: start level and the number
    of vectors scored for a query that sees the whole index are the pages'."""
    g = _golden(golden_dir)
    rng = np.random.default_rng(5)
    for key in ("lsa_tree_1m", "lsa_tree_10m"):
        f = g[key]
        P = f["tokens"] // 512 * 64
        assert P == f["buckets"]
        sizes_ = [P]
        while len(sizes_) < 4:
            sizes_.append(sizes_[-1] // f["node_block"] * (f["node_block"] // f["fanout"]))
        bits = [to_bf16_bits(rng.standard_normal((n, 64)) * 0.1) for n in sizes_]
        q = to_bf16_bits(rng.standard_normal((1, 64)))
        off = np.zeros(P + 1, dtype=np.int32)
        _, det = lsa_tree_levels_select(q, np.asarray([f["tokens"]]), bits[0], bits[1:], off,
                                        np.zeros(0, dtype=np.int32), 512, 64, f["node_block"], f["fanout"],
                                        f["beam"], f["start_nodes"], 4, 1024, 4096, return_detail=True)
        assert det[0]["start"] == f["start_level"]
        if "level1_nodes" in f:
            assert sizes_[1] == f["level1_nodes"]
        if "start_level_nodes" in f:
            assert sizes_[f["start_level"]] == f["start_level_nodes"]
        assert sum(det[0]["counts"].values()) == f["scored"], key


def test_lsa_generator_node_levels():
    """A level-2 node centroid is the normalised sum of the key sums of the 16
    buckets beneath it (size x centroid each): the levels sum keys, not
    normalised centroids."""
    d = make_workload("lsa_tree_levels_s")
    sizes_ = np.diff(d["bucket_off"]).astype(np.float64)
    c = bf16_to_f64(d["centroids"])
    n2 = bf16_to_f64(d["node_levels"][1])
    for j in (0, 1, 100, 287):
        s = (c[16 * j:16 * j + 16] * sizes_[16 * j:16 * j + 16, None]).sum(axis=0)
        assert np.allclose(n2[j], s / np.linalg.norm(s), atol=2 ** -8)


def test_two_stage_full_shortlist_equals_exact():
    d = make_two_stage(B=2, N=700, H=4, d=16, seed=8, plant_frac=0.05, ragged=100)
    n = d["n_valid"]
    got_i, got_v = two_stage_select(d["q"], d["w"], d["ck"], d["ck_scale"], d["fk"], d["fk_scale"], n,
                                    shortlist=700, k=32)
    for b in range(2):
        keys = dequant(d["fk"][b, : n[b]], d["fk_scale"][b, : n[b]], "e4m3")
        s = indexer_scores(bf16_to_f64(d["q"][b])[None], d["w"][b].astype(np.float64)[None], keys)[0]
        ei, ev = select_topk(s, np.arange(n[b]), 32)
        assert np.array_equal(got_i[b], ei)
        assert np.array_equal(got_v[b], ev)


def test_two_stage_brute_force_tiny():
    d = make_two_stage(B=1, N=60, H=2, d=8, seed=9, plant_frac=0.1)
    gi, gv, det = two_stage_select(d["q"], d["w"], d["ck"], d["ck_scale"], d["fk"], d["fk_scale"],
                                   d["n_valid"], shortlist=12, k=5, return_detail=True)
    qb = bf16_to_f64(d["q"][0]).tolist()
    wb = d["w"][0].astype(np.float64).tolist()
    ck = [[float(x) * float(d["ck_scale"][0, s]) for x in d["ck"][0, s]] for s in range(60)]
    fk = e4m3_to_f64(d["fk"][0]) * d["fk_scale"][0].astype(np.float64)[:, None]
    shat = [brute.score(qb, wb, ck[s]) for s in range(60)]
    short, _ = brute.topk(shat, list(range(60)), 12)
    ex = [brute.score(qb, wb, fk[s].tolist()) for s in short]
    bp, _ = brute.topk(ex, short, 5)
    assert gi[0].tolist() == bp
    assert det[0]["shortlist"].tolist() == short


def test_bucket_full_budget_equals_exact():
    d = make_bucket(T=3, clusters=50, cluster_size=8, H=4, d=16, seed=10, min_size=4, max_size=16)
    P = 50
    N = d["keys"].shape[0]
    gi, gv = bucket_select(d["q"], d["w"], d["centroids"], d["bucket_off"], d["bucket_mem"], d["keys"],
                           top_p=P, budget=N, k=64)
    ri, rv = decode_select(d["q"], d["w"], np.broadcast_to(d["keys"], (3,) + d["keys"].shape),
                           np.full(3, N), k=64)
    assert np.array_equal(gi, ri)
    assert np.array_equal(gv, rv)


def test_bucket_expansion_cuts_last_bucket():
    off = np.array([0, 3, 5, 9])
    mem = np.array([10, 11, 12, 20, 21, 30, 31, 32, 33])
    # picked order 2, 0, 1 with budget 6: all of bucket 2, then 2 of bucket 0
    assert expand_buckets([2, 0, 1], off, mem, 6).tolist() == [30, 31, 32, 33, 10, 11]
    assert expand_buckets([1, -1], off, mem, 6).tolist() == [20, 21]


def test_bucket_brute_force_tiny():
    d = make_bucket(T=2, clusters=12, cluster_size=8, H=2, d=8, seed=11, min_size=2, max_size=6)
    gi, gv, det = bucket_select(d["q"], d["w"], d["centroids"], d["bucket_off"], d["bucket_mem"], d["keys"],
                                top_p=4, budget=10, k=6, return_detail=True)
    cf = bf16_to_f64(d["centroids"]).tolist()
    kf = bf16_to_f64(d["keys"]).tolist()
    for t in range(2):
        qt = bf16_to_f64(d["q"][t]).tolist()
        wt = d["w"][t].astype(np.float64).tolist()
        cs = [brute.score(qt, wt, c) for c in cf]
        picked, _ = brute.topk(cs, list(range(12)), 4)
        cand = []
        for p in picked:
            for m in d["bucket_mem"][d["bucket_off"][p]: d["bucket_off"][p + 1]]:
                if len(cand) < 10:
                    cand.append(int(m))
        ex = [brute.score(qt, wt, kf[m]) for m in cand]
        bp, _ = brute.topk(ex, cand, 6)
        assert gi[t].tolist() == bp
        assert det[t]["cand"].tolist() == cand


def test_recall():
    assert recall_at_k(np.array([[1, 2, 3]]), np.array([[3, 2, 1]])) == 1.0
    assert recall_at_k(np.array([[1, 2, 9]]), np.array([[3, 2, 1]])) == pytest.approx(2 / 3)


def test_bucket_generator_centroid_is_member_mean():
    d = make_bucket(T=1, clusters=20, cluster_size=8, H=2, d=16, seed=12)
    kf = bf16_to_f64(d["keys"])
    for p in range(20):
        mem = d["bucket_mem"][d["bucket_off"][p]: d["bucket_off"][p + 1]]
        assert list(mem) == sorted(mem)
        mean = kf[mem].mean(axis=0)
        assert np.array_equal(d["centroids"][p], to_bf16_bits(mean))


# --------------------------------------------------------------------------- #
# the pages' printed figures
# --------------------------------------------------------------------------- #
def _golden(golden_dir):
    with open(os.path.join(golden_dir, "page_figures.json")) as f:
        return json.load(f)


def _close(got, fig):
    if "abs_tol" in fig:
        return abs(got - fig["value"]) <= fig["abs_tol"]
    return abs(got - fig["value"]) <= fig["rel_tol"] * abs(fig["value"]) + 1e-12


def test_page_figures(golden_dir):
    g = _golden(golden_dir)
    assert sizes.INDEXER_ENTRY_BYTES == g["indexer_entry_bytes"]["value"]
    assert sizes.KV_ENTRY_BYTES == g["kv_latent_entry_bytes"]["value"]
    f = g["indexer_mb_per_layer_128k"]
    assert _close(sizes.indexer_bytes(f["tokens"]) / 1e6, f)
    f = g["indexer_gb_61_layers_128k"]
    assert _close(f["layers"] * sizes.indexer_bytes(f["tokens"]) / 1e9, f)
    f = g["indexer_kflop_per_token_64_heads"]
    assert _close(sizes.indexer_flops_per_pair(f["heads"]) / 1e3, f)
    f = g["indexer_main_crossover_tokens"]
    assert _close(f["k"] * sizes.KV_ENTRY_BYTES / sizes.INDEXER_ENTRY_BYTES, f)
    f = g["prefill_history_load_ms"]
    assert _close(sizes.prefill_history_load_ms(f["tokens"], f["gbps"]), f)
    f = g["key_to_hot_buffer_ratio_512k"]
    assert _close(sizes.key_to_hot_buffer_ratio(f["tokens"]), f)
    h = sizes.lsa_holding(g["lsa_10m_buckets"]["tokens"])
    assert h["buckets"] == g["lsa_10m_buckets"]["value"]
    assert h["centroid_bytes"] == g["lsa_10m_centroid_mib"]["value"] * 2 ** 20
    assert h["member_bytes"] == g["lsa_10m_member_mib"]["value"] * 2 ** 20
    assert h["glm_keys"] == g["glm_10m_indexer_keys"]["value"]
    assert h["glm_key_bytes"] == g["glm_10m_indexer_key_mib"]["value"] * 2 ** 20


def test_ratio_readings():
    # 512K read as 512,000 tokens gives 7.16 (the printed 7.2); the binary
    # reading gives 7.33; without the 4 B scale the figures drop to 6.94 / 7.11.
    assert sizes.key_to_hot_buffer_ratio(512000) == pytest.approx(7.1615, abs=1e-3)
    assert sizes.key_to_hot_buffer_ratio(524288) == pytest.approx(7.3333, abs=1e-3)
    assert sizes.key_to_hot_buffer_ratio(512000, with_scale=False) == pytest.approx(6.944, abs=1e-3)
    assert abs(sizes.key_to_hot_buffer_ratio(512000) - 7.2) <= 0.05


# --------------------------------------------------------------------------- #
# sparse main attention over the selected rows
# --------------------------------------------------------------------------- #
from oracle.attention import default_scale, merge_partials, sparse_attention  # noqa: E402
from workloads.synth import make_attention  # noqa: E402


def _attn_case(T=3, H=4, N=40, k=12, d=24, seed=5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, d))
    lat = rng.standard_normal((N, d))
    idx = np.stack([rng.choice(N, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    return q, lat, idx


def test_attention_brute_force_tiny():
    q, lat, idx = _attn_case()
    idx[1, 7:] = -1
    idx[2, :] = -1
    scale, d_v = 0.3, 16
    o, lse = sparse_attention(q, lat, idx, scale, d_v)
    for t in range(q.shape[0]):
        rows = [list(lat[s]) for s in idx[t] if s >= 0]
        bo, bl = brute.attention([list(x) for x in q[t]], rows, scale, d_v)
        assert np.allclose(o[t], np.array(bo), rtol=1e-12, atol=1e-12)
        assert np.allclose(lse[t], np.array(bl), rtol=1e-12, atol=0) or (not rows and np.all(np.isneginf(lse[t])))
    assert np.all(o[2] == 0.0) and np.all(np.isneginf(lse[2]))


def test_attention_equals_dense_sdpa_when_every_row_is_selected():
    """Selecting every row reduces to dense attention of one query over the
    whole cache (MQA: every head attends to the same rows), computed here by
    torch's scaled_dot_product_attention in fp64."""
    q, lat, _ = _attn_case(T=2, H=3, N=50, d=32)
    scale, d_v = 0.17, 20
    idx = np.tile(np.arange(50, dtype=np.int32)[::-1], (2, 1))
    o, lse = sparse_attention(q, lat, idx, scale, d_v)
    qt = torch.from_numpy(q)[:, :, None, :]                                  # [T, H, 1, D]
    kt = torch.from_numpy(lat)[None, None].expand(2, 3, 50, 32)
    vt = torch.from_numpy(lat[:, :d_v])[None, None].expand(2, 3, 50, d_v)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, :, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)
    from scipy.special import logsumexp
    assert np.allclose(lse, logsumexp(scale * np.einsum("thd,nd->thn", q, lat), axis=2), rtol=1e-13)


def test_attention_closed_forms():
    q, lat, idx = _attn_case(T=2, H=3, N=30, k=9, d=16)
    scale = 0.5
    # one selected row: the output is that row's value part, lse its logit
    one = np.full_like(idx, -1)
    one[:, 4] = idx[:, 0]
    o, lse = sparse_attention(q, lat, one, scale, 10)
    for t in range(2):
        assert np.array_equal(o[t], np.tile(lat[idx[t, 0], :10], (3, 1)))
        assert np.allclose(lse[t], scale * q[t] @ lat[idx[t, 0]], rtol=1e-14)
    # a zero query: uniform weights, the mean of the selected values, lse = log n
    o, lse = sparse_attention(np.zeros_like(q), lat, idx, scale, 10)
    for t in range(2):
        assert np.allclose(o[t], np.tile(lat[idx[t]][:, :10].mean(axis=0), (3, 1)), rtol=1e-13, atol=1e-15)
        assert np.allclose(lse[t], math.log(9), rtol=1e-14)


def test_attention_invariants():
    """Slot order and where the unused slots sit do not matter; attention over
    a union of disjoint selections is the online-softmax merge of the parts."""
    q, lat, idx = _attn_case(T=3, H=4, N=60, k=20, d=24, seed=9)
    scale = 0.4
    o, lse = sparse_attention(q, lat, idx, scale, 16)
    rng = np.random.default_rng(1)
    perm = np.full((3, 27), -1, dtype=np.int32)
    for t in range(3):
        slots = rng.choice(27, size=20, replace=False)
        perm[t, slots] = rng.permutation(idx[t])
    o2, lse2 = sparse_attention(q, lat, perm, scale, 16)
    assert np.allclose(o2, o, rtol=1e-12, atol=1e-14) and np.allclose(lse2, lse, rtol=1e-13)
    a, b = idx.copy(), idx.copy()
    a[:, 8:] = -1
    b[:, :8] = -1
    oa, la = sparse_attention(q, lat, a, scale, 16)
    ob, lb = sparse_attention(q, lat, b, scale, 16)
    om, lm = merge_partials(oa, la, ob, lb)
    assert np.allclose(om, o, rtol=1e-12, atol=1e-14) and np.allclose(lm, lse, rtol=1e-13)
    # merging with an empty part changes nothing
    e = np.full_like(idx, -1)
    oe, le = sparse_attention(q, lat, e, scale, 16)
    om, lm = merge_partials(o, lse, oe, le)
    assert np.array_equal(om, o) and np.array_equal(lm, lse)


def test_attention_generator():
    d = make_attention(7, 16, 3000, 300, ragged=250)
    nv = (d["idx"] >= 0).sum(axis=1)
    assert nv[0] == 0 and nv[1] == 1 and np.all(nv[2:] >= 50)
    for t in range(7):   # distinct rows, a valid prefix
        row = d["idx"][t]
        assert np.all(row[:nv[t]] >= 0) and np.all(row[nv[t]:] == -1)
        assert len(set(row[:nv[t]].tolist())) == nv[t]
    lat = bf16_to_f64(d["latent"])
    assert abs(lat.std() - 1.0) < 0.01 and abs(default_scale() - 1 / 24) < 1e-15
