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


def test_attention_line_error_keeps_the_other_lines(monkeypatch):
    """The attention line runs last and an exception there is recorded in its
    own entry; the variants before it (the shard merge just before) are kept."""
    names = ["bench_prefill", "bench_bucket", "bench_lsa", "bench_lsa_tree", "bench_two_stage", "bench_shard_merge"]
    for n in names:
        monkeypatch.setattr(bench, n, lambda *a, **k: {"ms_per_step": 1.0})

    def boom(*a, **k):
        raise RuntimeError("attention failed")

    monkeypatch.setattr(bench, "bench_attention", boom)
    res = bench.bench_variants(None, None, {}, "measured")
    assert list(res)[-2:] == ["prefill_shard_merge", "attn_decode"]
    assert "attention failed" in res["attn_decode"]["error"]
    assert all(v == {"ms_per_step": 1.0} for k, v in res.items() if k != "attn_decode")
    with pytest.raises(RuntimeError):                       # asked for alone, it fails loudly
        bench.bench_variants(None, None, {}, "measured", only="attn_decode")
