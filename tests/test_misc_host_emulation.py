"""The bucket search's expansion kernel and the causal eligible-count kernel,
compiled for the host (no GPU).

`expand_kernel` (`csrc/misc.cuh`, one warp per query) lists the members of a
query's picked buckets in pick order, each bucket's members in stored order,
until the budget is held, and pads the rest with -1; a warp prefix sum over 32
picks at a time places each bucket.  `causal_counts_kernel` gives a query at
position t the number of stride-compressed keys it may see.  The source is
preprocessed (launchers removed; the shim supplies the warp shuffles) and
built with g++ under AddressSanitizer.  Expected values: the oracle's
`expand_buckets` (the -1 tail past its list) and `eligible_count`, exactly.
`fold_scales_kernel` (the fp8 path's head weight times query-head scale, a
grid-stride loop) is checked against numpy's fp32 product, bit for bit, with
grids smaller and larger than the array.
Picked lists end in a -1 tail where fewer buckets were found, as the top-k
writes them.  Test infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

from oracle.indexer import eligible_count
from oracle.select import expand_buckets

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc", "misc.cuh")


def _host_source() -> str:
    with open(SRC) as f:
        src = f.read()
    parts = []
    for name in ("causal_counts_kernel", "fold_scales_kernel", "expand_kernel"):
        m = re.search(r"__global__ void " + name + r"\(.*?\n\}\n", src, flags=re.S)
        assert m, name
        parts.append(m.group(0))
    return '#pragma once\n#include "cuda_shim.h"\nnamespace lsi {\n' + "".join(parts) + "}\n"


@pytest.fixture(scope="module")
def misc_host(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("misc_host")
    (d / "misc_host.h").write_text(_host_source())
    exe, env = host_build(d, "misc_host", "misc_main.cpp")

    def run(args):
        r = subprocess.run([str(exe), str(d)] + [str(a) for a in args], capture_output=True, text=True, env=env,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-3000:]

    return d, run


def _csr(sizes, rng):
    off = np.zeros(sizes.size + 1, dtype=np.int32)
    np.cumsum(sizes, out=off[1:])
    mem = rng.permutation(max(int(off[-1]), 1))[: int(off[-1])].astype(np.int32)
    for p in range(sizes.size):                          # members stored ascending within a bucket
        mem[off[p]: off[p + 1]].sort()
    return off, mem


EXPAND_CASES = ["bucket_workload", "ragged", "one_bucket_fills", "budget_above_all"]


@pytest.mark.parametrize("case", EXPAND_CASES)
def test_expand(misc_host, case):
    d, run = misc_host
    rng = np.random.default_rng(EXPAND_CASES.index(case))
    if case == "bucket_workload":                       # 32768 buckets of 8 keys, top 64, 512 keys
        P, top_p, budget, T = 32768, 64, 512, 40
        sizes = np.full(P, 8)
    elif case == "ragged":                              # empty and large buckets, top_p off the warp width
        P, top_p, budget, T = 500, 45, 300, 37
        sizes = rng.integers(0, 41, size=P)
        sizes[rng.choice(P, 60, replace=False)] = 0
    elif case == "one_bucket_fills":                    # the first pick alone overflows the budget
        P, top_p, budget, T = 64, 33, 100, 9
        sizes = rng.integers(90, 400, size=P)
    else:                                               # fewer members in all than the budget
        P, top_p, budget, T = 300, 70, 4000, 11
        sizes = rng.integers(0, 9, size=P)
    off, mem = _csr(sizes, rng)
    picked = np.full((T, top_p), -1, dtype=np.int32)
    for t in range(T):
        n = top_p - (t % 5) * (top_p // 7)              # some lists end early
        picked[t, :n] = rng.choice(P, n, replace=False)
    picked.tofile(d / "picked.bin")
    off.tofile(d / "off.bin")
    mem.tofile(d / "mem.bin")
    run(["expand", T, top_p, P, budget])
    cand = np.fromfile(d / "cand.bin", dtype=np.int32).reshape(T, budget)
    for t in range(T):
        want = expand_buckets(picked[t], off, mem, budget)
        assert np.array_equal(cand[t, : want.size], want.astype(np.int32)), t
        assert np.all(cand[t, want.size:] == -1), t


@pytest.mark.parametrize("stride,n_total", [(4, 8192), (1, 1000), (4, 5), (16, 70000)])
def test_causal_counts(misc_host, stride, n_total):
    d, run = misc_host
    rng = np.random.default_rng(stride * 7 + n_total)
    edge = stride * n_total
    pos = np.concatenate([[-1, 0, 1, stride - 2, stride - 1, stride, edge - 2, edge - 1, edge, edge + 1, 3 * edge],
                          rng.integers(0, 2 * edge + 2, 600)]).astype(np.int64)
    pos = pos[pos >= -1]
    pos.tofile(d / "pos.bin")
    run(["counts", pos.size, stride, n_total])
    cnt = np.fromfile(d / "cnt.bin", dtype=np.int32)
    assert np.array_equal(cnt, eligible_count(pos, stride, n_total).astype(np.int32))


@pytest.mark.parametrize("n,blocks", [(1, 1), (1000, 2), (70000, 3), (300, 8)])
def test_fold_scales(misc_host, n, blocks):
    d, run = misc_host
    rng = np.random.default_rng(n)
    w = rng.standard_normal(n).astype(np.float32)
    qs = np.abs(rng.standard_normal(n)).astype(np.float32) * np.float32(0.01)
    w.tofile(d / "w.bin")
    qs.tofile(d / "qs.bin")
    run(["fold", n, blocks])
    out = np.fromfile(d / "out.bin", dtype=np.float32)
    assert np.array_equal(out.view(np.uint32), (w * qs).view(np.uint32))
