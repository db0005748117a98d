"""The sampled-threshold reading of the LSA search (no GPU).

The threshold form is exact whatever the threshold (a row whose list holds
its top_p is exact, any other row is scored in full), so its threshold is a
matter of cost, not of correctness.  The reading: score every
(top_p / 16)-th visible bucket and take the 32nd best of those samples;
32 of 16 * v / top_p samples is a fraction 2 * top_p / v of the row, so
about 2 * top_p buckets should reach it, and a list of 4 * top_p rarely
overflows.  Checked here on the synthetic workloads in fp64: the mean list is
within 10% of 2 * top_p and no sampled row comes up short of its top_p or
overflows 4 * top_p (each such row would cost a full rescoring).
"""

import numpy as np
import pytest

from oracle.formats import bf16_to_f64
from oracle.select import lsa_visible
from workloads import get_workload, make_workload


@pytest.mark.parametrize("name", ["lsa_flat_s", "lsa_prefill_s", "lsa_flat"])
def test_lists_hold_about_twice_top_p(name):
    wl = get_workload(name)
    d = make_workload(name)
    cent, q = bf16_to_f64(d["centroids"]), bf16_to_f64(d["q_idx"])
    top_p, P = wl.top_p, cent.shape[0]
    vis = lsa_visible(d["q_pos"], wl.extra.get("block_keys", 512), wl.extra.get("buckets_per_block", 64), P)
    stride = max(1, top_p // 16)
    rows = np.arange(q.shape[0])
    if rows.size > 256:
        rows = np.random.default_rng(0).choice(rows, 256, replace=False)
    counts = []
    for t in rows:
        v = int(vis[t])
        scores = cent[:v] @ q[t]
        samples = scores[::stride]
        if samples.size < 32:                 # too few samples: the row is scored in full
            continue
        thr = np.sort(samples)[::-1][31]
        c = int((scores >= thr).sum())
        assert min(top_p, v) <= c <= 4 * top_p, (t, c)
        counts.append(c)
    assert len(counts) >= 20
    assert abs(np.mean(counts) / (2 * top_p) - 1) < 0.1, np.mean(counts)
