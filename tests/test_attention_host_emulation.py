"""The attention kernels' own source, compiled for the host and checked against the oracle (no GPU).

`csrc/sparse_attn.cuh` is preprocessed (launchers removed, its one packed-FMA
instruction mapped to two correctly rounded fused multiply-adds, the CUDA
features it uses supplied by `host_emulation/cuda_shim.h`) and built with g++ under
AddressSanitizer; each CUDA thread of a block runs as an OS thread, with real
barriers for `__syncthreads` and the warp shuffles.  This checks the kernels'
index arithmetic, staging, barriers, softmax and combine on every CPU run,
and any out-of-bounds access to the inputs, outputs or shared memory.  It
says nothing about timing or the GPU's own rounding of exp/log (the GPU
tests do).  Test infrastructure only: the product has no host path.
"""

import os
import re
import subprocess

import numpy as np
import pytest

from oracle.attention import default_scale, merge_partials, sparse_attention
from oracle.formats import bf16_to_f64
from workloads import make_workload
from workloads.synth import make_attention

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc", "sparse_attn.cuh")
TOL = 1e-4


def _host_source(src: str) -> str:
    src = src.replace('#include "common.cuh"', '#include "cuda_shim.h"')
    src = re.sub(r"cudaError_t launch_\w+\(.*?\n}\n", "", src, flags=re.S)
    src = src.replace("extern __shared__ __align__(16) unsigned char attn_smem[];",
                      "unsigned char* attn_smem = ::g_smem;")
    fma2 = 'asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));'
    assert fma2 in src
    src = src.replace(fma2, "acc = host_fma2(acc, a, b);")
    assert "<<<" not in src and "asm(" not in src and "attn_smem = ::g_smem" in src
    return src


@pytest.fixture(scope="module")
def runner(tmp_path_factory, host_build):
    d = tmp_path_factory.mktemp("attn_host")
    with open(SRC) as f:
        (d / "kernel_host.h").write_text(_host_source(f.read()))
    exe, env = host_build(d, "attn_host", "attn_main.cpp", ubsan=False)

    def attn(q, lat, idx, scale, off=None, foreign=False):
        T, H, _ = q.shape
        q.astype(np.uint16).tofile(d / "q.bin")
        lat.astype(np.uint16).tofile(d / "lat.bin")
        idx.astype(np.int32).tofile(d / "idx.bin")
        if off is not None:
            off.astype(np.int64).tofile(d / "off.bin")
        r = subprocess.run([str(exe), "attn", str(d), str(T), str(H), str(idx.shape[1]), str(lat.shape[0]),
                            repr(float(scale)), "1" if off is not None else "0", "1" if foreign else "0"],
                           capture_output=True, text=True, env=env, timeout=600)
        assert r.returncode == 0, r.stderr[-3000:]
        out = np.fromfile(d / "out.bin", dtype=np.float32).reshape(T, H, 512)
        lse = np.fromfile(d / "lse.bin", dtype=np.float32).reshape(T, H)
        return out, lse, int(r.stdout.strip())

    def merge(o_parts, lse_parts):
        S, dv = o_parts.shape[0], o_parts.shape[-1]
        rows = lse_parts[0].size
        o_parts.astype(np.float32).tofile(d / "op.bin")
        lse_parts.astype(np.float32).tofile(d / "lp.bin")
        r = subprocess.run([str(exe), "merge", str(d), str(S), str(rows), str(dv), "3"], capture_output=True,
                           text=True, env=env, timeout=600)
        assert r.returncode == 0, r.stderr[-3000:]
        return (np.fromfile(d / "mo.bin", dtype=np.float32).reshape(o_parts.shape[1:]),
                np.fromfile(d / "ml.bin", dtype=np.float32).reshape(lse_parts.shape[1:]))

    return attn, merge


def _compare(out, lse, q, lat, gidx, scale):
    ro, rl = sparse_attention(bf16_to_f64(q), bf16_to_f64(lat), gidx, scale)
    latf = bf16_to_f64(lat)
    for t in range(q.shape[0]):
        sel = gidx[t][gidx[t] >= 0]
        if sel.size == 0:
            assert np.all(out[t] == 0.0) and np.all(np.isneginf(lse[t])), t
            continue
        vmax = np.abs(latf[sel, :512]).max()
        assert np.abs(out[t] - ro[t]).max() <= TOL * vmax, t
        assert np.all(np.abs(lse[t] - rl[t]) <= TOL * (1 + np.abs(rl[t]))), t


def test_host_kernel_small_ragged_and_scattered(runner):
    attn, _ = runner
    d = make_workload("attn_s")
    out, lse, fault = attn(d["q"], d["latent"], d["idx"], default_scale())
    assert fault == 0
    _compare(out, lse, d["q"], d["latent"], d["idx"], default_scale())
    rng = np.random.default_rng(3)
    idx = np.stack([rng.permutation(r) for r in d["idx"]])
    out, lse, _ = attn(d["q"], d["latent"], idx, default_scale())
    _compare(out, lse, d["q"], d["latent"], idx, default_scale())


def test_host_kernel_row_offsets_bad_rows_and_shards(runner):
    attn, _ = runner
    d = make_workload("attn_s")
    N = d["latent"].shape[0]
    idx = np.where(d["idx"] >= 0, d["idx"] % 1000, -1).astype(np.int32)
    off = np.array([0, 10, 2000, 1500, 0, 2999, 5], dtype=np.int64)
    out, lse, fault = attn(d["q"], d["latent"], idx, 0.07, off)
    g = np.where(idx >= 0, idx + off[:, None], -1)
    bad = (idx >= 0) & (g >= N)
    assert bad.any() and fault == 2
    _compare(out, lse, d["q"], d["latent"], np.where(bad, -1, g), 0.07)
    # one shard of the rows: other shards' rows are skipped without the fault
    base, length = 1200, 900
    off = np.full(d["q"].shape[0], -base, dtype=np.int64)
    out, lse, fault = attn(d["q"], d["latent"][base:base + length], d["idx"], default_scale(), off, foreign=True)
    assert fault == 0
    local = np.where((d["idx"] >= base) & (d["idx"] < base + length), d["idx"] - base, -1)
    _compare(out, lse, d["q"], d["latent"][base:base + length], local, default_scale())


def test_host_kernel_long_selections_and_many_heads(runner):
    attn, _ = runner
    for T, H, N, k in ((1, 8, 5000, 2048), (1, 24, 3000, 130), (1, 8, 6000, 4612)):
        d = make_attention(T, H, N, k, seed=k)
        out, lse, fault = attn(d["q"], d["latent"], d["idx"], default_scale())
        assert fault == 0
        _compare(out, lse, d["q"], d["latent"], d["idx"], default_scale())


def test_host_merge_kernel(runner):
    _, merge = runner
    rng = np.random.default_rng(5)
    o = rng.standard_normal((3, 2, 8, 512)).astype(np.float32)
    lse = (rng.standard_normal((3, 2, 8)) * 3).astype(np.float32)
    lse[1, 0] = -np.inf
    lse[:, 1, 3] = -np.inf
    mo, ml = merge(o, lse)
    ro, rl = o[0].astype(np.float64), lse[0].astype(np.float64)
    for s in (1, 2):
        ro, rl = merge_partials(ro, rl, o[s].astype(np.float64), lse[s].astype(np.float64))
    assert np.all(mo[1, 3] == 0.0) and np.isneginf(ml[1, 3])
    assert np.abs(mo - ro).max() <= 1e-5 * np.abs(o).max()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(ml), np.isneginf(rl))
    assert np.all(np.abs(ml[fin] - rl[fin]) <= 1e-5 * (1 + np.abs(rl[fin])))
