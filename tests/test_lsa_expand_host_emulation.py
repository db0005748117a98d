"""The LSA read-list kernel, compiled for the host (no GPU), against the oracle's read list.

`lsa_expand_kernel` (`csrc/score_dot.cuh`) writes each query's sinks below
its window, the window, then the picked buckets' members best first (members
in the sinks or the window skipped) until `budget` long-range keys are held,
copying a round's members block-wide through a binary search over the
round's bucket starts.  Its source is preprocessed (static shared arrays
become function statics: the emulator runs one CTA at a time) and built with
g++ under AddressSanitizer, each CUDA thread an OS thread with real barriers.
Cases: the edge positions of the reduced LSA index (no visible block, sinks
inside the window, the first visible block), picks that are buckets of block
0 (members in the sinks), padded picks, more than one round of 1024 picks,
and budgets that cut a bucket.  Expected: `oracle.select.lsa_read_list`,
exactly.  Test infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

from oracle.select import lsa_read_list
from workloads import make_workload

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc")


def _host_source() -> str:
    with open(os.path.join(CSRC, "score_dot.cuh")) as f:
        dot = f.read()
    m = re.search(r"__device__ __forceinline__ int lower_bound_i32\(.*?\n\}\n", dot, flags=re.S)
    assert m
    parts = [m.group(0)]
    m = re.search(r"constexpr int kExpandThreads = 256;\nconstexpr int kExpandItems = 4;\n\n"
                  r"__global__ void __launch_bounds__\(kExpandThreads\)\n    lsa_expand_kernel\(.*?\n\}\n", dot, flags=re.S)
    assert m
    parts.append(m.group(0).replace("__shared__ ", "static "))
    return '#pragma once\n#include "cuda_shim.h"\nnamespace lsi {\n' + "".join(parts) + "}\n"


@pytest.fixture(scope="module")
def expand_host(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("lsa_expand_host")
    (d / "lsa_expand_host.h").write_text(_host_source())
    exe, env = host_build(d, "lsa_expand_host", "lsa_expand_main.cpp")
    return d, exe, env


@pytest.mark.parametrize("top_p,budget", [(64, 512), (1500, 4096), (300, 37)])
def test_read_lists_match_the_oracle(expand_host, top_p, budget):
    d, exe, env = expand_host
    w = make_workload("lsa_flat_s")
    off, mem, q_pos = w["bucket_off"], w["bucket_mem"], w["q_pos"].copy()
    P = off.size - 1
    T = q_pos.size
    rng = np.random.default_rng(top_p + budget)
    picked = np.full((T, top_p), -1, dtype=np.int32)
    for t in range(T):
        vis = min(int(q_pos[t]) // 512 * 64, P)
        take = min(vis, top_p - (t % 3) * 7)                 # some rows padded at the end
        if take > 0:
            picked[t, :take] = rng.permutation(vis)[:take]
    picked[1, :8] = np.arange(8)                             # block-0 buckets: members in the sinks
    d_ = d
    picked.tofile(d_ / "picked.bin")
    q_pos.astype(np.int64).tofile(d_ / "qpos.bin")
    off.astype(np.int32).tofile(d_ / "off.bin")
    mem.astype(np.int32).tofile(d_ / "mem.bin")
    r = subprocess.run([str(exe), str(d_), str(T), str(top_p), str(P), str(mem.size), "512", "4", str(budget)],
                       capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    row = 4 + 512 + budget
    keys = np.fromfile(d_ / "keys.bin", dtype=np.int32).reshape(T, row)
    n = np.fromfile(d_ / "n.bin", dtype=np.int32)
    for t in range(T):
        want = lsa_read_list(picked[t], q_pos[t], off, mem, 512, 4, budget)
        assert n[t] == want.size and np.array_equal(keys[t, :n[t]], want), t
        assert np.all(keys[t, n[t]:] == -1), t
