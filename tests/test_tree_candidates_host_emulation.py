"""The LSA tree search's candidate-scoring and level-visibility kernels, compiled
for the host (no GPU).

`lsa_tree_candidates_kernel` (`csrc/score_tree.cuh`) lists a query's
candidates at one level -- the children of its beam (nodes of the level
above, -1 padding past the visible ones), then the level's visible entries
that no node covers -- and scores each as its centroid's 64-d dot product
with the index query.  Its source is preprocessed (the packed FMA through the
shim's host version, the static shared query row a function static: the
emulator runs one CTA at a time) and built with g++ under AddressSanitizer.
Inputs: the three-level reduced index's level-1 centroids with level-2 beams
(full, partial and empty), and the bucket level with level-1 beams.
Expected: the candidate labels in that order, exactly, and scores within
fp32 rounding of the oracle's fp64 dot products.

`lsa_tree_levels_visible_kernel` gives each query its visible entry count at
every level: complete key blocks at the bucket level, complete node blocks
above, each capped by the level's size.  Expected: the oracle's
`lsa_visible` and `lsa_tree_levels`, exactly, for positions at and around
every block edge.  The one-level tree's visibility kernel and the flat
search's (which also counts the sampled buckets below the visible count, every
stride-th from bucket 0) are checked the same way.  Test infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

from oracle.formats import bf16_to_f64
from oracle.select import lsa_tree_levels, lsa_visible
from workloads import get_workload, make_workload

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc")


def _host_source() -> str:
    with open(os.path.join(CSRC, "score_tree.cuh")) as f:
        src = f.read()
    parts = []
    with open(os.path.join(CSRC, "score_dot.cuh")) as f:
        m = re.search(r"__global__ void lsa_visible_kernel\(.*?\n\}\n", f.read(), flags=re.S)
    assert m, "lsa_visible_kernel"
    parts.append(m.group(0))
    for pat in (r"__global__ void lsa_tree_visible_kernel\(.*?\n\}\n",
                r"struct TreeLevels \{.*?\n\};\n",
                r"__global__ void lsa_tree_levels_visible_kernel\(.*?\n\}\n",
                r"__device__ __forceinline__ float dot64_bf16\(.*?\n\}\n",
                r"__global__ void __launch_bounds__\(256\)\n    lsa_tree_candidates_kernel\(.*?\n\}\n"):
        m = re.search(pat, src, flags=re.S)
        assert m, pat
        parts.append(m.group(0))
    body = "".join(parts).replace("__shared__ ", "static ")
    fma = 'asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc[e]) : "l"(cw), "l"(q2[4 * v + e]));'
    assert fma in body
    body = body.replace(fma, "acc[e] = host_fma2(acc[e], cw, q2[4 * v + e]);")
    assert "asm(" not in body
    return ('#pragma once\n#include "cuda_shim.h"\nnamespace lsi {\nconstexpr int kLsaDim = 64;\nconstexpr int kMaxTreeLevels = 16;\n' + body + "}\n")


@pytest.fixture(scope="module")
def cand_host(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("tree_cand_host")
    (d / "tree_cand_host.h").write_text(_host_source())
    exe, env = host_build(d, "tree_cand_host", "tree_candidates_main.cpp")
    return d, exe, env


@pytest.mark.parametrize("level", [0, 1])
def test_candidates_and_scores(cand_host, level):
    d, exe, env = cand_host
    wl = get_workload("lsa_tree_levels_s")
    ex = wl.extra
    data = make_workload("lsa_tree_levels_s")
    fan, blk, beam_w = ex["fanout"], ex["node_block"], 24
    levels = [data["centroids"]] + list(data["node_levels"])
    sizes = [x.shape[0] for x in levels]
    q = data["q_idx"]
    T = q.shape[0]
    vis0 = lsa_visible(data["q_pos"], 512, 64, sizes[0])
    rng = np.random.default_rng(level)
    beam = np.full((T, beam_w), -1, dtype=np.int32)
    vis = np.zeros(T, np.int32)
    visn = np.zeros(T, np.int32)
    for t in range(T):
        v = lsa_tree_levels(vis0[t], sizes[1:], blk, fan)
        vis[t], visn[t] = v[level], v[level + 1]
        nb = min(beam_w, v[level + 1]) - (t % 4 == 1) * 3         # some beams shorter than the visible nodes
        if nb > 0:
            beam[t, :nb] = rng.permutation(v[level + 1])[:nb]
    cap = beam_w * fan + blk
    c = levels[level]
    q.astype(np.uint16).tofile(d / "q.bin")
    c.astype(np.uint16).tofile(d / "c.bin")
    beam.tofile(d / "beam.bin")
    vis.tofile(d / "vis.bin")
    visn.tofile(d / "visn.bin")
    r = subprocess.run([str(exe), str(d), str(T), str(c.shape[0]), str(beam_w), str(fan), str(cap)],
                       capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    cval = np.fromfile(d / "cval.bin", dtype=np.float32).reshape(T, cap)
    clab = np.fromfile(d / "clab.bin", dtype=np.int32).reshape(T, cap)
    nv = np.fromfile(d / "nv.bin", dtype=np.int32)
    cf = bf16_to_f64(c)
    for t in range(T):
        nb = min(beam_w, int(visn[t]))
        labs = [int(beam[t, i // fan]) * fan + i % fan if beam[t, i // fan] >= 0 else -1 for i in range(nb * fan)]
        labs += list(range(fan * int(visn[t]), int(vis[t])))
        assert nv[t] == len(labs), t
        assert np.array_equal(clab[t, :nv[t]], np.asarray(labs, dtype=np.int32)), t
        ok = np.asarray(labs) >= 0
        ref = cf[np.asarray(labs)[ok]] @ bf16_to_f64(q[t]) if ok.any() else np.zeros(0)
        got = cval[t, :nv[t]][ok]
        assert np.allclose(got, ref, rtol=1e-5, atol=1e-6), t
        assert np.all(np.isneginf(cval[t, :nv[t]][~ok])), t


@pytest.mark.parametrize("shape", [(512, 64, 4096, 4, [5000, 1248, 312, 76]),
                                   (512, 64, 4096, 4, [40960, 10240, 2560]),
                                   (128, 16, 256, 2, [3000, 1500, 700, 300, 100, 40])])
def test_level_visibility(cand_host, shape):
    d, exe, env = cand_host
    block_keys, bpb, blk, fan, sizes = shape
    n_keys = sizes[0] // bpb * block_keys
    edges = np.arange(0, n_keys + 3 * block_keys, block_keys, dtype=np.int64)
    rng = np.random.default_rng(len(sizes))
    pos = np.concatenate([edges - 1, edges, edges + 1, rng.integers(0, n_keys + 2 * block_keys, 700),
                          np.asarray([0, 1, (blk // bpb) * block_keys - 1, (blk // bpb) * block_keys])]).astype(np.int64)
    pos = pos[pos >= 0]
    T = pos.shape[0]
    pos.tofile(d / "pos.bin")
    args = [str(exe), str(d), "vis", str(T), str(block_keys), str(bpb), str(blk), str(fan), str(len(sizes) - 1)]
    r = subprocess.run(args + [str(x) for x in sizes], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.fromfile(d / "lvis.bin", dtype=np.int32).reshape(len(sizes), T)
    vis0 = lsa_visible(pos, block_keys, bpb, sizes[0])
    for t in range(T):
        want = lsa_tree_levels(int(vis0[t]), sizes[1:], blk, fan)
        assert list(got[:, t]) == list(want), (t, int(pos[t]))


def _edge_positions(block_keys, n_keys, node_span, seed):
    edges = np.arange(0, n_keys + 3 * block_keys, block_keys, dtype=np.int64)
    if edges.size > 1500:                              # long histories: every few edges, the first and the last
        edges = np.unique(np.concatenate([edges[:64], edges[::edges.size // 1000], edges[-64:]]))
    rng = np.random.default_rng(seed)
    pos = np.concatenate([edges - 1, edges, edges + 1, rng.integers(0, n_keys + 2 * block_keys, 700),
                          np.asarray([-5, -block_keys - 1, -3 * block_keys, 0, 1, node_span - 1, node_span])]).astype(np.int64)   # negative positions are clamped to 0
    return pos


@pytest.mark.parametrize("shape", [(512, 64, 5000, 4096, 4, 1248), (512, 64, 131072, 4096, 4, 32768),
                                   (128, 16, 3000, 256, 2, 700)])
def test_one_level_visibility(cand_host, shape):
    d, exe, env = cand_host
    block_keys, bpb, P, blk, fan, P1 = shape
    pos = _edge_positions(block_keys, P // bpb * block_keys, (blk // bpb) * block_keys, P)
    pos.tofile(d / "pos.bin")
    T = pos.size
    r = subprocess.run([str(exe), str(d), "vis1", str(T), str(block_keys), str(bpb), str(P), str(blk), str(fan), str(P1)],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.fromfile(d / "lvis.bin", dtype=np.int32).reshape(2, T)
    vis0 = lsa_visible(pos, block_keys, bpb, P)
    assert np.array_equal(got[0], vis0.astype(np.int32))
    want = [lsa_tree_levels(int(v), [P1], blk, fan)[1] for v in vis0]
    assert np.array_equal(got[1], np.asarray(want, dtype=np.int32))


@pytest.mark.parametrize("shape", [(512, 64, 131072, 64), (512, 64, 1310720, 64), (128, 16, 3000, 1), (512, 64, 5000, 7)])
def test_flat_visibility_and_sample_counts(cand_host, shape):
    d, exe, env = cand_host
    block_keys, bpb, P, stride = shape
    pos = _edge_positions(block_keys, P // bpb * block_keys, block_keys, stride)
    pos.tofile(d / "pos.bin")
    T = pos.size
    r = subprocess.run([str(exe), str(d), "visflat", str(T), str(block_keys), str(bpb), str(P), str(stride)],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.fromfile(d / "lvis.bin", dtype=np.int32).reshape(2, T)
    vis0 = lsa_visible(pos, block_keys, bpb, P)
    assert np.array_equal(got[0], vis0.astype(np.int32))
    assert np.array_equal(got[1], np.asarray([len(range(0, int(v), stride)) for v in vis0], dtype=np.int32))
