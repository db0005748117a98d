"""ls_decode_select_noalloc: decode selection for callers that cannot allocate.

Some callers cannot give the library a workspace (an engine that owns the
whole device pool, a loop that cannot afford cudaMalloc's synchronisation).
This entry point keeps its scratch in a fixed device array inside the
library.  The test calls it through the C ABI twice in a row, on two different
problems, and checks each result against ls_decode_select with a workspace;
it also checks that a problem too large for the fixed scratch is refused.
The file is named to be collected last, and passes alone or after the rest.
"""

import ctypes

import numpy as np
import pytest
import torch

from parity_util import dev, dev_bf16
from workloads.synth import make_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_lightning_b200 import build
    build.build()
    from sparse_attention_indexer_lightning_b200 import _lib
    return _lib.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _with_workspace(lib, q, w, k, nv, kk, stream):
    B, H, d = q.shape
    N = k.shape[1]
    ws = torch.empty(max(1, lib.ls_decode_select_workspace_size(B, N)), dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, kk), dtype=torch.int32, device="cuda")
    val = torch.empty((B, kk), dtype=torch.float32, device="cuda")
    st = lib.ls_decode_select(_p(q), _p(w), _p(k), _p(nv), B, H, d, N, kk, _p(idx), _p(val), _p(ws), ws.numel(),
                              stream)
    assert st == 0, lib.ls_last_error()
    return idx, val


def _noalloc(lib, q, w, k, nv, kk, stream):
    B, H, d = q.shape
    N = k.shape[1]
    idx = torch.full((B, kk), 7, dtype=torch.int32, device="cuda")
    val = torch.full((B, kk), 7.0, dtype=torch.float32, device="cuda")
    st = lib.ls_decode_select_noalloc(_p(q), _p(w), _p(k), _p(nv), B, H, d, N, kk, _p(idx), _p(val), stream)
    assert st == 0, lib.ls_last_error()
    return idx, val


def test_noalloc_matches_workspace_call_twice(lib):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        make_decode(B=6, N=5000, seed=41, ragged=900),        # ragged rows, several tiles
        make_decode(B=3, N=20000, seed=42, n_valid=np.array([20000, 300, 12345])),
    ]
    for d in cases:  # two calls in a row; the second sees the first one's leftovers
        q, w, k, nv = dev_bf16(d["q"]), dev(d["w"]), dev_bf16(d["k"]), dev(d["n_valid"])
        i0, v0 = _noalloc(lib, q, w, k, nv, 512, stream)
        i1, v1 = _with_workspace(lib, q, w, k, nv, 512, stream)
        torch.cuda.synchronize()
        i0, v0, i1, v1 = (t.cpu().numpy() for t in (i0, v0, i1, v1))
        # the same kernels on the same inputs: indices and values bit for bit
        assert np.array_equal(i0, i1)
        assert np.array_equal(v0.view(np.uint32), v1.view(np.uint32))


def test_noalloc_refuses_oversized_problem(lib):
    dummy = ctypes.c_void_p(256)
    # 64 x 65536 scores need 16 MiB of scratch, more than the fixed array
    st = lib.ls_decode_select_noalloc(dummy, dummy, dummy, None, 64, 32, 128, 65536, 512, dummy, None, None)
    assert st == 2  # LS_ERR_WORKSPACE
    assert b"fixed scratch" in lib.ls_last_error()
