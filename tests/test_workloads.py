"""The seeded synthetic inputs (no GPU).  The oracle and the CUDA path read
the same generated arrays, and every stored expectation is regenerated from
a seed, so a workload must come out byte for byte the same for a seed, and
differently for another."""

import numpy as np
import pytest

from workloads import get_workload, make_workload

SMALL = ["decode_tiny", "decode_s", "prefill_s", "prefill_fp8_s", "two_stage_s", "two_stage_pq_s", "lsa_flat_s",
         "lsa_tree_levels_s", "lsa_prefill_s", "attn_s", "bucket_s"]


def _arrays(d, prefix=""):
    for k, v in sorted(d.items()):
        if isinstance(v, np.ndarray):
            yield prefix + k, v
        elif isinstance(v, (list, tuple)):
            for i, x in enumerate(v):
                if isinstance(x, np.ndarray):
                    yield f"{prefix}{k}[{i}]", x


@pytest.mark.parametrize("name", SMALL)
def test_same_seed_same_bytes(name):
    a, b = dict(_arrays(make_workload(name))), dict(_arrays(make_workload(name)))
    assert a.keys() == b.keys() and a
    for k in a:
        assert a[k].dtype == b[k].dtype and a[k].shape == b[k].shape, k
        assert a[k].tobytes() == b[k].tobytes(), k


@pytest.mark.parametrize("name", SMALL)
def test_other_seed_other_values(name):
    wl = get_workload(name)
    a, b = dict(_arrays(make_workload(name))), dict(_arrays(make_workload(name, seed=wl.seed + 1)))
    assert a.keys() == b.keys()
    assert any(a[k].tobytes() != b[k].tobytes() for k in a)
    for k in a:                                       # only the values move: shapes and dtypes are the workload's
        assert a[k].dtype == b[k].dtype, k
