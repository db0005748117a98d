"""Back-to-back calls of the streamed prefill selection, as a serving loop and
the benchmark make them: one workspace, one pair of tile buffers and one copy
stream reused by every call, with no host synchronisation between calls.

The workspace starts filled with 0xFF bytes, so any read of a workspace word
that the call has not written yet sees NaN / -1 patterns instead of a
previous call's leftovers.  Each call writes its own output buffers; every
call's selection must equal the full-matrix form's bit for bit, that form must
pass the band rule against the oracle, and the library's device fault word
must stay clear.  Cases: the small chunk workload (several tiles, a ragged
last tile), a chunk with k = 32 (many filtered candidates per tile), queries
whose scores rise with position (every later tile overflows the candidate
slots of half the rows: the full-tile fallback), and a 600-query chunk whose
merge rows take the four-CTAs-per-SM top-k form the benchmark's chunk uses.
The LSA sampled-threshold search gets the same treatment (one workspace,
0xFF-filled, ten calls, bit-equal to its full-matrix form), with and without
every row falling back.
"""

from types import SimpleNamespace

import numpy as np
import pytest
import torch

from oracle.formats import bf16_to_f64, dequant
from oracle.indexer import eligible_count, indexer_scores
from parity_util import RTOL_BF16, RTOL_FP8, check_selection, dev, dev_bf16
from workloads import get_workload, make_workload
from workloads.synth import make_prefill, quantize_e4m3_rows, to_bf16_bits

pytestmark = pytest.mark.gpu

CALLS = 20


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_lightning_b200 import build as b
    b.build()
    import sparse_attention_indexer_lightning_b200 as lib
    return lib


def _rising(fp8: bool):
    """Half the queries point along the keys' direction, whose length rises
    with position: each later tile beats their whole running list."""
    T, H, dd, N, stride = 24, 32, 128, 1000, 4
    rng = np.random.default_rng(7)
    u = rng.standard_normal(dd)
    u /= np.linalg.norm(u)
    alpha = np.linspace(0.05, 1.0, N)
    kf = alpha[:, None] * u[None, :]
    sign = np.where(np.arange(T) < T // 2, 1.0, -1.0)
    qf = np.broadcast_to(sign[:, None, None] * u[None, None, :], (T, H, dd)).copy()
    d = {"q": to_bf16_bits(qf), "k": to_bf16_bits(kf),
         "w": (np.abs(rng.standard_normal((T, H))) + 0.1).astype(np.float32),
         "q_pos": (stride * N - 1 - rng.integers(0, 300, size=T)).astype(np.int64)}
    if fp8:
        d["q8"], d["q_scale"] = quantize_e4m3_rows(qf)
        d["k8"], d["k_scale"] = quantize_e4m3_rows(kf)
    return d, SimpleNamespace(k=32, stride=stride, tile_keys=128)


def _case(name: str, fp8: bool):
    if name == "small":
        wl = get_workload("prefill_fp8_s" if fp8 else "prefill_s")
        return make_workload(wl), wl
    if name == "small_k32":
        return make_prefill(77, 1019, 4000, seed=3, fp8=fp8), SimpleNamespace(k=32, stride=4, tile_keys=256)
    if name == "rising":
        return _rising(fp8)
    # 600 queries (more than twice the SMs: the 256-thread top-k form), 5.9 tiles
    return make_prefill(600, 6000, 4 * 6000 - 600, seed=11, fp8=fp8), SimpleNamespace(k=512, stride=4,
                                                                                        tile_keys=1024)


class _Runner:
    """Device inputs, host history, buffers and a copy stream for one case."""

    def __init__(self, L, d, wl, fp8: bool):
        self.L, self.wl, self.fp8 = L, wl, fp8
        self.w, self.qp = dev(d["w"]), dev(d["q_pos"])
        if fp8:
            self.q8, self.qs = dev(d["q8"]), dev(d["q_scale"])
            self.hk = torch.from_numpy(np.ascontiguousarray(d["k8"])).pin_memory()
            self.hs = torch.from_numpy(np.ascontiguousarray(d["k_scale"])).pin_memory()
            self.bufs = [torch.empty(wl.tile_keys * 132, dtype=torch.uint8, device="cuda") for _ in range(2)]
            self.T, self.N = d["q8"].shape[0], d["k8"].shape[0]
        else:
            self.q = dev_bf16(d["q"])
            self.hk = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
            self.bufs = [torch.empty((wl.tile_keys, 128), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
            self.T, self.N = d["q"].shape[0], d["k"].shape[0]
        self.cs = torch.cuda.Stream()

    def ws_bytes(self, full: bool) -> int:
        f = (self.L.lib().ls_prefill_select_fp8_workspace_size if self.fp8
             else self.L.lib().ls_prefill_select_workspace_size)
        return f(self.T, self.N, self.wl.tile_keys, self.wl.k, int(full))

    def call(self, full: bool, ws, out):
        wl = self.wl
        if self.fp8:
            return self.L.ls_prefill_select_stream_fp8(self.q8, self.qs, self.w, self.qp, self.hk, self.hs,
                                                       self.bufs[0], self.bufs[1], k=wl.k, stride=wl.stride,
                                                       tile_keys=wl.tile_keys, full_scores=full, ws=ws, out=out,
                                                       copy_stream=self.cs)
        return self.L.ls_prefill_select_stream(self.q, self.w, self.qp, self.hk, self.bufs[0], self.bufs[1],
                                               k=wl.k, stride=wl.stride, tile_keys=wl.tile_keys, full_scores=full,
                                               ws=ws, out=out, copy_stream=self.cs)


def _oracle_scores(d, t, n, fp8):
    if fp8:
        return indexer_scores(dequant(d["q8"][t], d["q_scale"][t], "e4m3")[None],
                              d["w"][t].astype(np.float64)[None], dequant(d["k8"][:n], d["k_scale"][:n], "e4m3"))[0]
    return indexer_scores(bf16_to_f64(d["q"][t])[None], d["w"][t].astype(np.float64)[None], bf16_to_f64(d["k"][:n]))[0]


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "fp8"])
@pytest.mark.parametrize("case", ["small", "small_k32", "rising", "wide"])
def test_prefill_running_repeated_calls(L, case, fp8):
    d, wl = _case(case, fp8)
    r = _Runner(L, d, wl, fp8)
    T, k = r.T, wl.k
    assert L.ls_device_status() == 0
    # reference: the full-matrix form, once, on its own workspace
    ws_full = torch.empty(r.ws_bytes(True), dtype=torch.uint8, device="cuda")
    ref_i, ref_v = r.call(True, ws_full, None)
    torch.cuda.synchronize()
    ref_i, ref_v = ref_i.cpu().numpy(), ref_v.cpu().numpy()
    del ws_full
    n_t = eligible_count(d["q_pos"], wl.stride, r.N)
    rtol = RTOL_FP8 if fp8 else RTOL_BF16
    rows = range(T) if T <= 100 else (0, 1, 2, 7, 8, 299, 300, T - 2, T - 1)
    for t in rows:
        n = int(n_t[t])
        check_selection(ref_i[t], ref_v[t], np.arange(n), _oracle_scores(d, t, n, fp8), k, rtol,
                        f"{case} full-matrix t={t}")
    # the running form, CALLS times back to back on one workspace (pre-filled
    # with 0xFF), one pair of buffers and one copy stream
    ws = torch.full((r.ws_bytes(False),), 0xFF, dtype=torch.uint8, device="cuda")
    outs = [(torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
             torch.full((T, k), 7.0, dtype=torch.float32, device="cuda")) for _ in range(CALLS)]
    torch.cuda.synchronize()
    for o in outs:
        r.call(False, ws, o)
    torch.cuda.synchronize()
    assert L.ls_device_status() == 0
    for c, (oi, ov) in enumerate(outs):
        gi, gv = oi.cpu().numpy(), ov.cpu().numpy()
        same = (gi == ref_i).all(axis=1) & f32_bits_equal_rows(gv, ref_v)
        assert same.all(), f"{case} call {c}: {int((~same).sum())} rows differ from the full-matrix form, " \
                           f"first row {int(np.flatnonzero(~same)[0])}"


def f32_bits_equal_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
            == np.ascontiguousarray(b, dtype=np.float32).view(np.uint32)).all(axis=1)


@pytest.mark.parametrize("case", ["plain", "all_fall_back"])
def test_lsa_threshold_repeated_calls(L, case):
    """Back-to-back calls of the LSA sampled-threshold search on the
    3000-query chunk with one workspace (0xFF-filled first) and one set of
    output buffers: every call's picks and read lists equal the full-matrix
    form's bit for bit and the fault word stays clear.  The second case makes
    every row miss its threshold (all centroids and queries along one
    direction, so every visible bucket ties), which runs the device-listed
    fallback in 256-row chunks on every call."""
    wl = get_workload("lsa_prefill_s")
    d = dict(make_workload("lsa_prefill_s"))
    ex = wl.extra
    if case == "all_fall_back":
        rng = np.random.default_rng(4)
        u = rng.standard_normal(64)
        u /= np.linalg.norm(u)
        d["q_idx"] = to_bf16_bits(np.broadcast_to(u, d["q_idx"].shape).copy())
        d["centroids"] = to_bf16_bits(np.broadcast_to(u, d["centroids"].shape).copy())
    fb_rows = 256 if case == "all_fall_back" else 0
    args = (dev_bf16(d["q_idx"]), dev(d["q_pos"]), dev_bf16(d["centroids"]), dev(d["bucket_off"]),
            dev(d["bucket_mem"]))
    kw = dict(block_keys=ex["block_keys"], buckets_per_block=ex["bpb"], n_sink=ex["n_sink"], top_p=wl.top_p,
              budget=wl.budget, want_picked=True)
    k0, n0, p0 = L.ls_lsa_flat_select(*args, threshold=False, **kw)
    T, P = d["q_idx"].shape[0], d["centroids"].shape[0]
    need = L.lib().ls_lsa_flat_workspace_size(T, P, wl.top_p, 1, fb_rows)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    row = ex["n_sink"] + ex["block_keys"] + wl.budget
    out = (torch.empty((T, row), dtype=torch.int32, device="cuda"), torch.empty((T,), dtype=torch.int32, device="cuda"))
    L.ls_device_status()
    results = []
    for _ in range(10):
        keys, n, picked = L.ls_lsa_flat_select(*args, threshold=True, fallback_rows=fb_rows, ws=ws, out=out, **kw)
        results.append((keys.clone(), n.clone(), picked.clone()))
    torch.cuda.synchronize()
    for i, (keys, n, picked) in enumerate(results):
        assert torch.equal(picked, p0) and torch.equal(n, n0) and torch.equal(keys, k0), f"call {i}"
    assert L.ls_device_status() == 0
