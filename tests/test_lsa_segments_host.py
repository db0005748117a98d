"""The LSA threshold scan's list-segment arithmetic, checked on the host (no GPU).

`kernels.h`'s `lsa_first_cta`, `lsa_segment` and `lsa_max_segments` are
shared by the scan kernel (where a CTA appends a row's listed buckets), the
compaction kernel (which packs a row's segments) and the workspace sizing.
A host program compiled by nvcc from the same header walks every query
group of a range of shapes (one group and all CTAs, many groups and a few
CTAs each, ragged tails, a grid smaller than the SM count) and checks that
the segments of a row tile its list in CTA order, stay inside the reserved
row width and index counters below nseg.  Test infrastructure only.
"""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "sparse_attention_indexer_lightning_b200", "csrc")

# (T, P, cap2, SM count)
SHAPES = [(1, 128, 32, 148), (37, 4992, 1024, 148), (256, 131072, 16384, 148), (257, 129, 64, 148),
          (3000, 32768, 4096, 148), (5000, 300, 1024, 148), (32768, 128, 8192, 148), (32768, 1310720, 8192, 148),
          (4096, 1310720, 8192, 148), (100000, 4096, 512, 148), (777, 77777, 2048, 132), (65536, 65536, 4096, 148)]


@pytest.fixture(scope="module")
def seg_bin(tmp_path_factory):
    nvcc = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else None)
    if nvcc is None:
        pytest.skip("no nvcc")
    d = tmp_path_factory.mktemp("seg")
    exe = d / "seg"
    r = subprocess.run([nvcc, "-std=c++17", "-O1", "-I", CSRC, "-I", os.path.join(os.path.dirname(HERE), "include"),
                        "-o", str(exe), os.path.join(HERE, "host_emulation", "segments_main.cu")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    return exe


def test_segments_tile_each_row(seg_bin):
    args = [str(x) for shape in SHAPES for x in shape]
    r = subprocess.run([str(seg_bin)] + args, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
