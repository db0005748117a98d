"""The shard-merge pack kernel's source, compiled for the host (no GPU).

`csrc/merge.cuh` is preprocessed (launchers removed, its static shared
variable a static local, the CUDA features it uses supplied by
`host_emulation/cuda_shim.h`) and built with g++ under AddressSanitizer,
each CUDA thread an OS thread with real barriers.  The packed rows must hold
every shard's valid prefix, in shard order, with the shard's first position
added, and the row counts.  Test infrastructure only.
"""

import os
import re
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc", "merge.cuh")


def _host_source(src: str) -> str:
    src = src.replace('#include "common.cuh"', '#include "cuda_shim.h"').replace('#include "kernels.h"', "")
    src = re.sub(r"cudaError_t launch_\w+\(.*?\n}\n", "", src, flags=re.S)
    src = src.replace("__shared__ int first_pad;", "static int first_pad;")
    assert "<<<" not in src and "static int first_pad;" in src
    return src


@pytest.fixture(scope="module")
def pack(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("merge_host")
    with open(SRC) as f:
        (d / "merge_host.h").write_text(_host_source(f.read()))
    exe, env = host_build(d, "merge_host", "merge_main.cpp", ubsan=False)

    def run(vals, idx, offs):
        S, T, k_in = vals.shape
        vals.astype(np.float32).tofile(d / "vals.bin")
        idx.astype(np.int32).tofile(d / "idx.bin")
        offs.astype(np.int32).tofile(d / "offs.bin")
        r = subprocess.run([str(exe), str(d), str(S), str(T), str(k_in)], capture_output=True, text=True, env=env,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-3000:]
        return (np.fromfile(d / "pv.bin", dtype=np.float32).reshape(T, S * k_in),
                np.fromfile(d / "pl.bin", dtype=np.int32).reshape(T, S * k_in),
                np.fromfile(d / "nv.bin", dtype=np.int32))

    return run


@pytest.mark.parametrize("S,T,k_in", [(1, 3, 40), (3, 5, 300), (4, 2, 600)])
def test_host_merge_pack(pack, S, T, k_in):
    rng = np.random.default_rng(S * 100 + k_in)
    vals = np.full((S, T, k_in), -np.inf, dtype=np.float32)
    idx = np.full((S, T, k_in), -1, dtype=np.int32)
    for s in range(S):
        for t in range(T):
            n = [0, k_in, 1, int(rng.integers(0, k_in + 1))][(s + t) % 4]
            idx[s, t, :n] = rng.integers(0, 5000, size=n)
            vals[s, t, :n] = rng.standard_normal(n)
    offs = np.arange(S, dtype=np.int32) * 5000
    pv, pl, nv = pack(vals, idx, offs)
    for t in range(T):
        ev, el = [], []
        for s in range(S):
            n = int((idx[s, t] >= 0).sum())
            ev.append(vals[s, t, :n])
            el.append(idx[s, t, :n] + offs[s])
        ev, el = np.concatenate(ev), np.concatenate(el)
        assert nv[t] == ev.size
        assert np.array_equal(pl[t, :ev.size], el)
        assert np.array_equal(pv[t, :ev.size].view(np.uint32), ev.view(np.uint32))
