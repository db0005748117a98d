"""The running prefill selection's segment-pack kernel, compiled for the host (no GPU).

`csrc/misc.cuh` is preprocessed (its launchers removed, the CUDA features the
pack kernel uses supplied by `host_emulation/cuda_shim.h`) and built with g++
under AddressSanitizer, each CUDA thread an OS thread with real barriers.
Each row holds the first tile's top-k in columns [0, k) and one segment of
`cap` candidate slots per later tile; the kernel moves, in place, every row's
present entries to one prefix: the k first-tile entries, then each segment's
first min(count, cap) entries (k when the row overflowed that tile).  Rows
here use shifts larger and smaller than the 256-entry chunk, empty and full
segments, overflowed segments, and a first segment already in place.  Test
infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc", "misc.cuh")


def _host_source(src: str) -> str:
    m = re.search(r"constexpr int kPackThreads = 256;\n.*?\n}\n", src, flags=re.S)
    assert m, "pack kernel not found"
    return ('#pragma once\n#include "cuda_shim.h"\nnamespace lsi {\n'
            + m.group(0).replace("__launch_bounds__(kPackThreads)", "") + "}\n")


@pytest.fixture(scope="module")
def pack(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("pack_host")
    with open(SRC) as f:
        (d / "pack_host.h").write_text(_host_source(f.read()))
    exe, env = host_build(d, "pack_host", "pack_main.cpp")

    def run(val, lab, cnt, over, k, cap):
        T, ld = val.shape
        S = cnt.shape[0]
        val.astype(np.float32).tofile(d / "val.bin")
        lab.astype(np.int32).tofile(d / "lab.bin")
        cnt.astype(np.uint32).tofile(d / "cnt.bin")
        over.astype(np.int32).tofile(d / "over.bin")
        r = subprocess.run([str(exe), str(d), str(T), str(ld), str(k), str(S), str(cap)], capture_output=True,
                           text=True, env=env, timeout=300)
        assert r.returncode == 0, r.stderr[-3000:]
        return (np.fromfile(d / "val.bin", dtype=np.float32).reshape(T, ld),
                np.fromfile(d / "lab.bin", dtype=np.int32).reshape(T, ld),
                np.fromfile(d / "nv.bin", dtype=np.int32))

    return run


@pytest.mark.parametrize("k,S", [(512, 3), (40, 5), (300, 1)])
def test_host_pack_segments(pack, k, S):
    cap = 2 * k
    ld = k + S * cap
    T = 12
    rng = np.random.default_rng(k + S)
    val = rng.standard_normal((T, ld)).astype(np.float32)
    lab = rng.integers(0, 10 ** 6, size=(T, ld)).astype(np.int32)
    cnt = rng.integers(0, cap + 1, size=(S, T)).astype(np.uint32)
    cnt[:, 0] = 0                               # every segment empty
    cnt[:, 1] = cap + 17                        # counted past the slots
    cnt[0, 2] = cap                             # a full first segment
    over = (rng.random((S, T)) < 0.2).astype(np.int32)
    over[:, 3] = 1                              # overflowed everywhere: k entries per segment
    want = []
    for t in range(T):
        parts_v, parts_l = [val[t, :k]], [lab[t, :k]]
        for j in range(S):
            n = k if over[j, t] else min(int(cnt[j, t]), cap)
            s0 = k + j * cap
            parts_v.append(val[t, s0:s0 + n])
            parts_l.append(lab[t, s0:s0 + n])
        want.append((np.concatenate(parts_v), np.concatenate(parts_l)))
    gv, gl, nv = pack(val.copy(), lab.copy(), cnt, over, k, cap)
    for t in range(T):
        wv, wl = want[t]
        assert nv[t] == wv.size
        assert np.array_equal(gl[t, :wv.size], wl)
        assert np.array_equal(gv[t, :wv.size].view(np.uint32), wv.view(np.uint32))
