"""Host logic of bench.py (no GPU): peaks, the roofline record, and the rule
that a DRAM-traffic figure from an ncu capture is reported only while the
kernel's sources are unchanged since the capture."""

import os

import pytest

import bench


def test_peaks_are_the_measured_file():
    peaks, kind = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured" and peaks["hbm_gbs"] > 1000
    else:
        assert kind == "fallback"


def test_roofline_record():
    r = bench.roofline("hbm", 5000.0, 6500.0, "GB/s", traffic=1.0e9)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 1.0e9
    assert r["frac"] == pytest.approx(5000.0 / 6500.0, abs=1e-4)


def test_traffic_only_for_unchanged_sources(monkeypatch):
    """Every row of the committed traffic table whose digest matches today's
    sources is reported; the same row under another digest is not."""
    rows = []
    with open(bench.TRAFFIC_FILE) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                rows.append(ln.rstrip("\n").split("\t"))
    assert rows
    for kernel, workload, nbytes, dig in rows:
        got = bench.ncu_traffic(kernel, workload)
        if bench.source_digest(kernel) == dig:
            assert got == float(nbytes)
        else:
            assert got is None
    kernel, workload = rows[0][0], rows[0][1]
    monkeypatch.setattr(bench, "source_digest", lambda k=None: "0000000000000000")
    assert bench.ncu_traffic(kernel, workload) is None


def test_digest_covers_the_kernel_sources():
    """A kernel listed with its sources hashes only those; one not listed
    hashes every CUDA source and the header (any change voids its figure)."""
    listed = bench.source_digest("score_tc_kernel<8>")
    assert listed == bench.source_digest("score_tc_kernel<1>")      # template arguments do not matter
    assert listed != bench.source_digest("dot_tc_kernel")
    assert bench.source_digest("topk_kernel") == bench.source_digest(None)


def test_variant_children_isolate_failures(monkeypatch):
    """Each variant runs in a child process; a child that dies (a sticky CUDA
    error ends its process), prints no line, or runs out of time leaves an
    error entry, and the variants after it still run."""
    import subprocess
    import types

    calls = []

    def fake_run(cmd, **kw):
        name = cmd[cmd.index("--only") + 1]
        calls.append(name)
        if name == "prefill_chunk_fp8_running":
            return types.SimpleNamespace(returncode=1, stdout="",
                                         stderr="torch.AcceleratorError: CUDA error: an illegal memory access")
        if name == "bucket":
            raise subprocess.TimeoutExpired(cmd, 1)
        if name == "lsa_flat":
            return types.SimpleNamespace(returncode=0, stdout="no json here\n", stderr="")
        return types.SimpleNamespace(returncode=0, stdout="log line\n" + bench.json.dumps(
            {"variant": name, name: {"ms_per_step": 1.0}}) + "\n", stderr="")

    monkeypatch.setattr(subprocess, "run", fake_run)
    args = types.SimpleNamespace(steps=3, warmup=3)
    names = ["prefill_chunk", "prefill_chunk_fp8_running", "bucket", "lsa_flat", "two_stage"]
    res = bench.bench_variants(args, names)
    assert calls == names
    assert res["prefill_chunk"]["ms_per_step"] == 1.0 and res["two_stage"]["ms_per_step"] == 1.0
    assert "illegal memory access" in res["prefill_chunk_fp8_running"]["error"]
    assert "timed out" in res["bucket"]["error"]
    assert "exit 0" in res["lsa_flat"]["error"]
    assert set(bench.DEFAULT_VARIANTS) <= set(bench.VARIANTS)


def test_reference_line(monkeypatch, capsys):
    """The reference arm's line: the oracle's rate on rank 0 only, the decode
    line's metric, unit and config, a cpu_baseline and an e2e equal to the
    line's value with no copies declared, and a step time that is one step of
    the workload (all its sequences) at that rate."""
    import types

    import numpy as np
    import workloads

    B, N, H, dd = 4, 1000, 32, 128
    tiny = {"q": np.zeros((B, H, dd), np.uint16), "w": np.zeros((B, H), np.float32),
            "k": np.zeros((B, N, dd), np.uint16)}
    monkeypatch.setattr(workloads, "make_workload", lambda wl, **kw: tiny)
    rates = iter([5.0e6, 9.0e6,                         # warm-up calls (ignored)
                  2.0e6, 3.0e6, 1.0e6] * 4)             # timed steps: the median is 2.0e6
    monkeypatch.setattr(bench, "oracle_decode_rate", lambda d, budget, k: (next(rates), 7, budget))
    monkeypatch.setattr(bench, "blas_threads", lambda: 8)
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.run_reference(types.SimpleNamespace(steps=3, warmup=2, workload="decode_batch")) == 0
    line = bench.json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] == 2.0e6 and line["unit"] == "positions/s"
    assert line["metric"].startswith("indexer query-positions scored/sec")
    assert line["ms_per_step"] == pytest.approx(B * N / 2.0e6 * 1e3)
    assert line["config"] == bench.decode_config(workloads.get_workload("decode_batch"), B, N, H, dd, 1)
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["cores"] == 8
    assert line["cpu_baseline"]["kind"] == "oracle" and "21 in total over 3 steps" in line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": 2.0e6, "unit": "positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # under torchrun the other ranks exit without work or output
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(types.SimpleNamespace(steps=3, warmup=2, workload="decode_batch")) == 0
    assert capsys.readouterr().out == ""
