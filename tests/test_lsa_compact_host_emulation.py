"""The LSA threshold form's compaction and missed-row list kernels, compiled for the host (no GPU).

`lsa_compact_kernel` packs each row's list segments (one per CTA of the scan
that scored the row, each in four quarters with their own counts) into one
list, and flags the rows whose list ran over or came up short;
`lsa_flag_list_kernel` lists the flagged rows in ascending order and marks
the fallback chunks that hold any; `lsa_gather_rows_kernel` copies the listed
rows' index queries and visible counts, in list order, into the fallback's
buffers (zeros past the count), and writes nothing while its run flag is
clear.  Their source in `csrc/score_dot.cuh` and
the segment arithmetic in `csrc/kernels.h` are preprocessed (static shared
arrays become function statics: the emulator runs one CTA at a time) and
built with g++ under AddressSanitizer, each CUDA thread an OS thread with real
barriers.  Inputs: segment contents and counts laid out as the scan writes
them, for one query group with every CTA and for many groups with a few
CTAs each, counts past a quarter's length (the scan's overflow), empty
quarters, short and long lists.  Expected: the segments' entries in quarter
order, the flags, the list, the chunk marks and the gathered rows, exactly.  Test
infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc")


def _host_source() -> str:
    with open(os.path.join(CSRC, "kernels.h")) as f:
        kern = f.read()
    with open(os.path.join(CSRC, "score_dot.cuh")) as f:
        dot = f.read()
    parts = []
    for pat in (r"struct LsaSeg \{.*?\n\};\n", r"__host__ __device__ inline int lsa_first_cta\(.*?\n\}\n",
                r"__host__ __device__ inline LsaSeg lsa_segment\(.*?\n\}\n"):
        m = re.search(pat, kern, flags=re.S)
        assert m, pat
        parts.append(m.group(0))
    for pat in (r"__global__ void __launch_bounds__\(256\)\n    lsa_compact_kernel\(.*?\n\}\n",
                r"__global__ void __launch_bounds__\(1024\)\n    lsa_flag_list_kernel\(.*?\n\}\n",
                r"__global__ void lsa_gather_rows_kernel\(.*?\n\}\n"):
        m = re.search(pat, dot, flags=re.S)
        assert m, pat
        parts.append(m.group(0).replace("__shared__ ", "static "))
    return ('#pragma once\n#include "cuda_shim.h"\nnamespace lsi {\nstruct DotCfg { static constexpr int QB = 256; };\n'
            'constexpr int kLsaDim = 64;\n'
            + "".join(parts) + "}\n")


def _segments(T, P, cap2, slack, grid_cap=148):
    """Python restatement of the layout: per row, per (j, q), (offset, length)."""
    NT = (P + 127) // 128
    G = (T + 255) // 256
    units = G * NT
    grid = min(units, grid_cap)
    per = max(1, units // grid)
    nseg = min(NT // per + 2, grid)
    out = {}
    for g in range(G):
        x = g * NT
        c0 = max(0, min(grid - 1, ((x + 1) * grid + units - 1) // units - 1))
        segs = []
        for j in range(nseg):
            c = c0 + j
            if c >= grid:
                break
            ub, ue = units * c // grid, units * (c + 1) // grid
            lo, hi = max(ub, x) - x, min(ue, x + NT) - x
            if hi <= lo:
                continue
            a, b = cap2 * lo // NT, cap2 * hi // NT
            off, ln = a + slack * j, b - a + slack
            for q in range(4):
                segs.append((j, q, off + q * (ln // 4), ln // 4))
        out[g] = segs
    return out, nseg, grid


@pytest.fixture(scope="module")
def compact_host(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("lsa_compact_host")
    (d / "lsa_compact_host.h").write_text(_host_source())
    exe, env = host_build(d, "lsa_compact_host", "lsa_compact_main.cpp")
    return d, exe, env


@pytest.mark.parametrize("T,P,top_p", [(37, 4992, 64), (600, 8192, 64), (300, 100000, 128)])
def test_compaction_and_missed_rows(compact_host, T, P, top_p):
    d, exe, env = compact_host
    rng = np.random.default_rng(T + P)
    cap = 4 * top_p
    cap2, slack = 2 * cap, 64
    segs, nseg, grid = _segments(T, P, cap2, slack)
    ld = cap2 + slack * nseg
    slist = np.zeros((T, ld, 2), dtype=np.uint32)
    slist[:, :, 0] = rng.integers(0, 2 ** 31, size=(T, ld), dtype=np.uint32)   # score bits
    slist[:, :, 1] = np.arange(ld, dtype=np.uint32)[None, :] + 100000 * np.arange(T, dtype=np.uint32)[:, None]
    cnt = np.zeros((T, nseg, 4), dtype=np.uint32)
    vis = rng.integers(0, 4 * top_p, size=T).astype(np.int32)
    want_val, want_lab, want_nv, want_over = [], [], np.zeros(T, np.int32), np.zeros(T, np.int32)
    for t in range(T):
        kind = t % 5
        quarters = segs[t // 256]
        # a row total around the list's size (short, in range, or too long),
        # spread over the quarters; kind 2 also runs one quarter past its end
        target = {0: 0, 1: int(rng.integers(0, top_p)), 2: int(rng.integers(top_p, cap)),
                  3: int(rng.integers(top_p, cap + 1)), 4: int(rng.integers(cap, 2 * cap))}[kind]
        share = rng.multinomial(target, np.full(len(quarters), 1.0 / len(quarters)))
        entries = []
        for i, (j, q, off, ln) in enumerate(quarters):
            n = int(min(share[i], ln))
            if kind == 2 and i == t % len(quarters):
                n = ln + int(rng.integers(1, 5))                 # ran past its quarter
            cnt[t, j, q] = n
            entries.extend(range(off, off + min(n, ln)))
        total = len(entries)
        want_nv[t] = min(total, cap)
        want_over[t] = int(total > cap or total < min(top_p, vis[t]))
        want_val.append(slist[t, entries, 0] if total <= cap else None)
        want_lab.append(slist[t, entries, 1] if total <= cap else None)
    q = rng.integers(0, 2 ** 16, size=(T, 64), dtype=np.uint16)
    slist.tofile(d / "slist.bin")
    cnt.tofile(d / "cnt.bin")
    vis.tofile(d / "vis.bin")
    q.tofile(d / "q.bin")
    rows = 50
    n_chunks = (T + rows - 1) // rows
    r = subprocess.run([str(exe), str(d), str(T), str(P), str(cap2), str(slack), str(nseg), str(grid), str(top_p),
                        str(cap), str(rows), str(n_chunks)], capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    cval = np.fromfile(d / "cval.bin", dtype=np.uint32).reshape(T, cap)
    clab = np.fromfile(d / "clab.bin", dtype=np.int32).reshape(T, cap)
    nv = np.fromfile(d / "nv.bin", dtype=np.int32)
    over = np.fromfile(d / "over.bin", dtype=np.int32)
    assert np.array_equal(nv, want_nv)
    assert np.array_equal(over[:T], want_over) and over[T] == int(want_over.any())
    for t in range(T):
        if want_val[t] is not None:
            n = want_val[t].size
            assert np.array_equal(cval[t, :n], want_val[t]), t
            assert np.array_equal(clab[t, :n], want_lab[t].astype(np.int32)), t
    flagged = np.flatnonzero(want_over)
    lst = np.fromfile(d / "list.bin", dtype=np.int32)
    count = int(np.fromfile(d / "count.bin", dtype=np.int32)[0])
    run = np.fromfile(d / "run.bin", dtype=np.int32)
    assert count == flagged.size
    assert np.array_equal(lst[:count], flagged) and np.all(lst[count:] == -1)
    assert np.array_equal(run, (np.arange(n_chunks) * rows < count).astype(np.int32))
    qbuf = np.fromfile(d / "qbuf.bin", dtype=np.uint16).reshape(T, 64)
    vbuf = np.fromfile(d / "vbuf.bin", dtype=np.int32)
    assert np.array_equal(qbuf[:count], q[flagged]) and np.all(qbuf[count:] == 0)
    assert np.array_equal(vbuf[:count], vis[flagged]) and np.all(vbuf[count:] == 0)
    assert np.all(np.fromfile(d / "qidle.bin", dtype=np.uint16) == 0x7777)
    assert np.all(np.fromfile(d / "vidle.bin", dtype=np.int32) == 777)
