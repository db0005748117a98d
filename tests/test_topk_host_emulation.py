"""The top-k kernel's own source, compiled for the host and checked against the oracle (no GPU).

`csrc/topk.cuh` is preprocessed (launchers removed, its dynamic shared block
mapped to a heap block of exactly the kernel's size, the few helpers it takes
from `common.cuh` and `kernels.h` copied in) and built with g++ under
AddressSanitizer and UndefinedBehaviorSanitizer (array-bounds checks on every
fixed-size shared array).  Each CUDA thread of a block runs as an OS thread,
with real barriers for `__syncthreads` and the warp collectives, so the OS
scheduler interleaves the threads in ways a GPU rarely does: a read of shared
memory that is not ordered by a barrier against another warp's writes shows
up as a wrong selection, a sanitizer report, or threads that disagree on a
branch around a barrier (a deadlock, ended by the timeout).

Rows cover every form the launcher picks (256 / 512 / 1024 threads), exact and
sampled histograms, the listed and the plain (whole-row radix) paths, labels
with absent entries (the merge rows of the running prefill top-k), n_valid
cuts, ties, NaN, +-inf and +-0.  Expected: the oracle's canonical top-k, bit
for bit.  Test infrastructure only: the product has no host path.
"""

import os
import re
import subprocess

import numpy as np
import pytest

from oracle.select import select_topk

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc")
FORMS = {0: (256, 512, 2048), 1: (512, 1024, 8192), 2: (1024, 4096, 8192)}


def _host_source() -> str:
    with open(os.path.join(CSRC, "common.cuh")) as f:
        common = f.read()
    with open(os.path.join(CSRC, "kernels.h")) as f:
        kern = f.read()
    with open(os.path.join(CSRC, "topk.cuh")) as f:
        topk = f.read()
    parts = []
    for pat, text in ((r"__device__ __forceinline__ uint32_t order_code\(float f\) \{.*?\n\}\n", common),
                      (r"constexpr int kHistBits = 11;\n", common),
                      (r"constexpr int kHistBins = 1 << kHistBits;\n", common),
                      (r"__device__ __forceinline__ uint32_t hist_bin\(uint32_t code\) \{[^\n]*\n", common),
                      (r"__device__ __forceinline__ float neg_inf\(\) \{[^\n]*\n", common),
                      (r"constexpr int kMaxTopK = \d+;\n", kern),
                      (r"struct TopkParams \{.*?\n\};\n", kern)):
        m = re.search(pat, text, flags=re.S)
        assert m, pat
        parts.append(m.group(0))
    body = topk.replace('#include "common.cuh"', "").replace('#include "kernels.h"', "").replace("#pragma once", "")
    body = re.sub(r"template <int NT, int KMAX, int CAP>\nstatic cudaError_t launch_topk_t\(.*?\n}\n", "", body,
                  flags=re.S)
    body = re.sub(r"cudaError_t launch_topk\(.*?\n}\n", "", body, flags=re.S)
    body = body.replace("extern __shared__ __align__(16) uint8_t topk_smem[];", "uint8_t* topk_smem = ::g_smem;")
    assert "<<<" not in body and "topk_smem = ::g_smem" in body
    return ('#pragma once\n#include "cuda_shim.h"\ntypedef void* cudaStream_t;\nnamespace lsi {\n' + "".join(parts)
            + "}\n" + body)


@pytest.fixture(scope="module")
def topk_host(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("topk_host")
    (d / "topk_host.h").write_text(_host_source())
    exe, env = host_build(d, "topk_host", "topk_main.cpp")

    def run(form, scores, labels, n_valid, k, flags=None, grid=0, out_row=None):
        R, ld = scores.shape
        scores.astype(np.float32).tofile(d / "scores.bin")
        if out_row is not None:
            out_row.astype(np.int32).tofile(d / "outrow.bin")
        elif (d / "outrow.bin").exists():
            (d / "outrow.bin").unlink()
        if labels is not None:
            labels.astype(np.int32).tofile(d / "labels.bin")
        if n_valid is not None:
            n_valid.astype(np.int32).tofile(d / "nvalid.bin")
        rows = [str(r) for r in range(R)]
        if flags is not None:
            flags.astype(np.int32).tofile(d / "flags.bin")
            rows = [str(-grid)]
        cmd = [str(exe), str(d), str(form), str(R), str(ld), str(k), str(ld), str(int(labels is not None)),
               str(int(n_valid is not None)), "0", "0", str(k)] + rows
        r = subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=300)
        assert r.returncode == 0, r.stderr[-3000:]
        return (np.fromfile(d / "idx.bin", dtype=np.int32).reshape(R, k),
                np.fromfile(d / "val.bin", dtype=np.float32).reshape(R, k))

    return run


def _row(rng, n, kind):
    if kind == "normal":
        return rng.standard_normal(n).astype(np.float32)
    if kind == "ties":                         # a handful of distinct values: the boundary bin is crowded
        return rng.integers(0, 8, n).astype(np.float32)
    if kind == "coarse":                       # quarter steps, like sums of fp8 products
        return (np.round(rng.standard_normal(n) * 4) / 4).astype(np.float32)
    if kind == "narrow":                       # one narrow cluster: a handful of the 2048 coarse bins
        return (0.3 + 1e-3 * rng.standard_normal(n)).astype(np.float32)
    if kind == "tail":                         # a long Gaussian row: the k-th entry deep in the tail
        return (0.125 * rng.standard_normal(n)).astype(np.float32)
    if kind == "special":
        v = rng.standard_normal(n).astype(np.float32)
        m = rng.integers(0, 6, n)
        v[m == 0], v[m == 1], v[m == 2], v[m == 3] = np.nan, -np.inf, 0.0, -0.0
        return v
    return np.full(n, 1.5, dtype=np.float32)   # one value: every key ties


def _merge_rows(rng, R, k):
    """Rows shaped like the running prefill top-k's merge: the running top-k
    (canonical order, padded with -1), then a tile's candidates."""
    ld = 4 * k
    sc = np.full((R, ld), np.nan, dtype=np.float32)
    lab = np.full((R, ld), -1, dtype=np.int32)
    nv = np.zeros(R, dtype=np.int32)
    for r in range(R):
        kind = ("normal", "coarse", "ties")[r % 3]
        run_v = np.sort(_row(rng, k, kind))[::-1]
        run_l = rng.permutation(8192)[:k].astype(np.int32)
        c = (0, 10, 600, 3 * k, 3 * k, 300, k, 2 * k)[r % 8]
        sc[r, :k], lab[r, :k] = run_v, run_l
        sc[r, k:k + c] = _row(rng, c, kind) + (r % 3)
        lab[r, k:k + c] = 8192 + rng.permutation(8192)[:c]
        if r % 8 == 5:
            lab[r, 100:k] = -1                 # a running list that was not full
        nv[r] = k + c
    return sc, lab, nv


def _expect(sc, lab, nv, k):
    R, ld = sc.shape
    out_i = np.empty((R, k), dtype=np.int64)
    out_v = np.empty((R, k), dtype=np.float32)
    for r in range(R):
        n = ld if nv is None else int(min(max(nv[r], 0), ld))
        pos = np.arange(n) if lab is None else lab[r, :n].astype(np.int64)
        keep = pos >= 0
        out_i[r], out_v[r] = select_topk(sc[r, :n][keep], pos[keep], k)
    return out_i, out_v


def _check(got, want):
    gi, gv = got
    wi, wv = want
    assert np.array_equal(gi, wi)
    assert np.array_equal(gv.view(np.uint32), wv.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("form,ld,k", [(0, 2048, 512), (0, 8192, 512), (0, 600, 512), (1, 9000, 1000),
                                       (2, 20000, 3000), (2, 3000, 4096)])
@pytest.mark.parametrize("labelled", [False, True])
def test_host_topk_rows(topk_host, form, ld, k, labelled):
    rng = np.random.default_rng(1000 * form + ld + k + int(labelled))
    R = 10
    kinds = ("normal", "ties", "coarse", "special", "const")
    sc = np.stack([_row(rng, ld, kinds[r % len(kinds)]) for r in range(R)])
    lab = None
    if labelled:
        lab = np.stack([rng.permutation(3 * ld)[:ld] for _ in range(R)]).astype(np.int32)
        lab[rng.random(lab.shape) < 0.1] = -1
    nv = rng.integers(0, ld + 1, R).astype(np.int32)
    nv[0], nv[1], nv[2] = ld, min(ld, k), 0
    _check(topk_host(form, sc, lab, nv, k), _expect(sc, lab, nv, k))


def test_host_topk_merge_rows(topk_host):
    """The running prefill top-k's merge rows, several times over (each run
    interleaves the threads differently)."""
    k = 512
    rng = np.random.default_rng(7)
    sc, lab, nv = _merge_rows(rng, 16, k)
    want = _expect(sc, lab, nv, k)
    for _ in range(3):
        _check(topk_host(0, sc, lab, nv, k), want)


def test_host_topk_flagged_rows_grid_stride(topk_host):
    """A launch with row flags walks the rows with fewer CTAs than rows: the
    flagged rows get their top-k, the others are left as they were."""
    k = 64
    rng = np.random.default_rng(11)
    R, ld = 13, 700
    sc = np.stack([_row(rng, ld, ("normal", "ties", "coarse")[r % 3]) for r in range(R)])
    nv = rng.integers(0, ld + 1, R).astype(np.int32)
    flags = (rng.random(R) < 0.5).astype(np.int32)
    flags[0], flags[R - 1] = 1, 1
    gi, gv = topk_host(0, sc, None, nv, k, flags=flags, grid=4)
    wi, wv = _expect(sc, None, nv, k)
    for r in range(R):
        if flags[r]:
            assert np.array_equal(gi[r], wi[r])
            assert np.array_equal(gv[r].view(np.uint32), wv[r].astype(np.float32).view(np.uint32))
        else:
            assert np.all(gi[r] == 777)          # untouched


def test_host_topk_out_row_map(topk_host):
    """With an output row map, row r's top-k lands in row out_row[r]; rows
    mapped to -1 write nothing, rows no input maps to are left as they were."""
    k = 64
    rng = np.random.default_rng(12)
    R, ld = 9, 500
    sc = np.stack([_row(rng, ld, ("normal", "ties", "coarse")[r % 3]) for r in range(R)])
    nv = rng.integers(0, ld + 1, R).astype(np.int32)
    out_row = np.array([3, -1, 0, 8, 1, -1, 2, 7, 4], dtype=np.int32)
    gi, gv = topk_host(0, sc, None, nv, k, out_row=out_row)
    wi, wv = _expect(sc, None, nv, k)
    for r in range(R):
        if out_row[r] >= 0:
            assert np.array_equal(gi[out_row[r]], wi[r])
            assert np.array_equal(gv[out_row[r]].view(np.uint32), wv[r].astype(np.float32).view(np.uint32))
    for o in set(range(R)) - set(out_row.tolist()):
        assert np.all(gi[o] == 777)


@pytest.mark.parametrize("form,ld,k", [(1, 200000, 1000), (2, 60000, 3000), (0, 50000, 512)])
def test_host_topk_long_rows_refined_boundary(topk_host, form, ld, k):
    """Long rows whose k-th entry sits in a coarse histogram bin (a narrow
    cluster, a deep Gaussian tail): the sampled boundary is refined by the next
    code bits so that the list fits, and the selection stays exact."""
    rng = np.random.default_rng(ld + k)
    R = 4
    sc = np.stack([_row(rng, ld, ("narrow", "tail")[r % 2]) for r in range(R)])
    nv = np.full(R, ld, dtype=np.int32)
    nv[3] = ld - 12345
    _check(topk_host(form, sc, None, nv, k), _expect(sc, None, nv, k))
