"""Benchmark of the lightning-indexer selection path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_batch] [--no-variants] [--variants default|all|A,B]
                    [--only NAME] [--no-cpu-baseline]

One step is one decode selection over the batch workload: 64 sequences x
32768 stride-4 compressed bf16 keys (131072 tokens each), 32 heads x 128 dims,
exact top-512 per sequence -- the scan (ls_indexer_score) then the selection
(ls_topk_select).  Inputs (537 MB of keys) are larger than the 126 MB L2, so
no flush is needed between steps.  The metric is query-positions scored per
second (selections per second alongside).  The prefill, two-stage, bucket
and LSA searches, and the sparse attention that follows a decode selection
(`attn_decode`), are timed the same way, each in a child process of its own
(`bench.py --only NAME`), and reported under "variants", each with the
roofline of its dominant kernel; a child that fails leaves an error entry and
the decode line is printed whatever the variants do.

With N > 1 (torchrun) every rank runs its own batch (weak scaling, no
collective on the data path); the reported time is the max over ranks.

--impl reference times the fp64 CPU oracle on this host's cores on a bounded
sample of the same workload (the oracle is the only reference this method
has).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------------------- #
# clocks sampler (nvidia-smi during the timed region)
# --------------------------------------------------------------------------- #
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread while the
    timed region runs (the region is short, so the polling is tight)."""

    REASONS = {  # NVML clocks-event-reason bits
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4,
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nvml = nv
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self._h = nv.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
            return
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = fn(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                break
            time.sleep(0.0001)

    def stop(self):
        if self._nvml is None:
            return None
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- #
# distributed plumbing
# --------------------------------------------------------------------------- #
def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun env).  backend "gloo" drives the same
    host logic on CPU (tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank time over all ranks (device tensor under NCCL)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's step time."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


# The device code each measured kernel's DRAM traffic depends on: its own
# source file, the shared device helpers and the parameter structs.
KERNEL_SOURCES = {
    "score_tc_kernel": ["common.cuh", "kernels.h", "score_tc.cuh"],
    "score_q8_kernel": ["common.cuh", "kernels.h", "score_q8.cuh"],
    "dot_tc_kernel": ["common.cuh", "kernels.h", "score_dot.cuh"],
    "sparse_attn_tc_kernel": ["common.cuh", "kernels.h", "sparse_attn_tc.cuh"],
}


def source_digest(kernel: str = None) -> str:
    """sha256 (first 16 hex digits) over the CUDA sources a kernel is built
    from (every CUDA source and the C header when the kernel is not listed):
    a DRAM-traffic figure taken from an ncu capture counts only while it matches."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_indexer_lightning_b200", "csrc")
    base = None if kernel is None else kernel.split("<")[0].split(":")[0]
    if base in KERNEL_SOURCES:
        files = [os.path.join(csrc, f) for f in KERNEL_SOURCES[base]]
    else:
        files = [os.path.join(csrc, f) for f in sorted(os.listdir(csrc))]
        files.append(os.path.join(ROOT, "include", "ls_indexer.h"))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload`, from the
    ncu table in profiles/, or None when absent or taken from other sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    dig = source_digest(kernel)
    for ln in lines:
        if not ln.strip() or ln.startswith("#"):
            continue
        parts = ln.split("\t")
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[3] == dig:
            return float(parts[2])
    return None


def roofline(bound, achieved, peak, unit, traffic=None, peak_kind="measured"):
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind}


def time_loop(fn, steps, warmup, stream, marks=None):
    """Run fn(step) warmup+steps times; returns (total_ms over the timed steps, per-mark ms sums)."""
    import torch
    for i in range(warmup):
        fn(i, None)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    ev = []
    start.record(stream)
    for i in range(steps):
        pair = fn(i, True)
        if pair is not None:
            ev.append(pair)
    end.record(stream)
    torch.cuda.synchronize()
    total = start.elapsed_time(end)
    seg = {}
    for pair in ev:
        for name, (a, b) in pair.items():
            seg[name] = seg.get(name, 0.0) + a.elapsed_time(b)
    return total, seg


def decode_config(wl, B, N, H, dd, world):
    """The decode workload's `config` entry, the same on both arms."""
    return {"workload": wl.name, "sequences_per_gpu": B, "compressed_positions": N, "tokens_per_sequence": 4 * N,
            "heads": H, "d": dd, "k": wl.k, "parallelism": f"replicas x{world}",
            "l2": f"inputs ({B * N * dd * 2 / 1e6:.0f} MB keys) larger than the 126 MB L2; no flush"}


def bench_decode(L, args, world, rank, peaks, peak_kind):
    import torch
    from workloads import get_workload, make_workload
    wl = get_workload(args.workload)
    d = make_workload(wl, seed=wl.seed + rank)
    B, H, dd = d["q"].shape
    N = d["k"].shape[1]
    q, w, k = to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev_bf16(d["k"])
    q4, w3 = q.view(B, 1, H, dd), w.view(B, 1, H)
    st = torch.cuda.current_stream()
    idx = torch.empty((B, wl.k), dtype=torch.int32, device="cuda")
    val = torch.empty((B, wl.k), dtype=torch.float32, device="cuda")
    lib = L.lib()
    import ctypes
    P = ctypes.c_void_p
    stp = P(st.cuda_stream)
    ws = torch.empty(lib.ls_decode_select_workspace_size(B, N), dtype=torch.uint8, device="cuda")

    def step(i, timed):
        s = lib.ls_decode_select(P(q.data_ptr()), P(w.data_ptr()), P(k.data_ptr()), None, B, H, dd, N, wl.k,
                                 P(idx.data_ptr()), P(val.data_ptr()), P(ws.data_ptr()), ws.numel(), stp)
        if s:
            raise RuntimeError(lib.ls_last_error().decode())
        return None

    clocks = ClockSampler(torch.cuda.current_device())
    for i in range(args.warmup):
        step(i, None)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    # the library brackets each of its kernel launches with CUDA events on the
    # launch stream while profiling is on: per-kernel time over the timed region
    L.ls_profile_begin()
    total_ms, _ = time_loop(step, args.steps, 0, st)
    prof = L.ls_profile_end()
    clk = clocks.stop()
    barrier(world)
    ms_per_step = max_over_ranks(total_ms / args.steps, world)
    scan_ms = prof["score_tc_kernel<1>"][0] / prof["score_tc_kernel<1>"][1]
    topk_ms = prof["topk_kernel"][0] / prof["topk_kernel"][1]
    launches = sum(c for _, c in prof.values())
    positions = B * N
    value = weak_scaling_value(positions, ms_per_step, world)
    key_bytes = B * N * dd * 2
    out = {
        "metric": "indexer query-positions scored/sec (decode selection, top-512)",
        "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(d) keys and queries, N(0,1)/sqrt(H) head weights)",
        "config": decode_config(wl, B, N, H, dd, world),
        "selections_per_s": world * B / (ms_per_step * 1e-3),
        "breakdown_ms": {"scan": scan_ms, "topk": topk_ms},
        "kernels": {kname: {"total_ms": v[0], "launches": v[1]} for kname, v in prof.items()},
        "roofline": roofline("hbm", key_bytes / (scan_ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                             traffic=ncu_traffic("score_tc_kernel<1>", wl.name), peak_kind=peak_kind),
        "gpu_launches": launches,
        "clocks": clk,
    }
    out["roofline"]["kernel"] = "score_tc_kernel<1> (decode scan)"
    out["roofline"]["algorithmic_bytes_per_launch"] = key_bytes
    # end to end through the C ABI with host buffers: copy the step's inputs in
    # from pinned memory, select, copy the selection back
    hq = torch.from_numpy(d["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hw = torch.from_numpy(d["w"]).pin_memory()
    hk = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    oi = torch.empty((B, wl.k), dtype=torch.int32).pin_memory()
    ov = torch.empty((B, wl.k), dtype=torch.float32).pin_memory()
    def e2e_step(i, timed):
        q.copy_(hq, non_blocking=True)
        w.copy_(hw, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        s = lib.ls_decode_select(P(q.data_ptr()), P(w.data_ptr()), P(k.data_ptr()), None, B, H, dd, N, wl.k,
                                 P(idx.data_ptr()), P(val.data_ptr()), P(ws.data_ptr()), ws.numel(), stp)
        if s:
            raise RuntimeError(lib.ls_last_error().decode())
        oi.copy_(idx, non_blocking=True)
        ov.copy_(val, non_blocking=True)
        return None

    e2e_steps = max(3, min(args.steps, 10))
    barrier(world)
    e2e_ms, _ = time_loop(e2e_step, e2e_steps, 2, st)
    e2e_ms = max_over_ranks(e2e_ms / e2e_steps, world)
    h2d = hq.numel() * 2 + hw.numel() * 4 + hk.numel() * 2
    d2h = oi.numel() * 4 + ov.numel() * 4
    out["e2e"] = {"value": world * positions / (e2e_ms * 1e-3), "unit": "positions/s", "ms_per_step": e2e_ms,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    return out, d


VARIANTS = {
    "prefill_chunk": lambda *a: bench_prefill(*a),
    "prefill_chunk_running": lambda *a: bench_prefill(*a, full_scores=False),
    "prefill_chunk_fp8": lambda *a: bench_prefill(*a, fp8=True),
    "prefill_chunk_fp8_running": lambda *a: bench_prefill(*a, full_scores=False, fp8=True),
    "bucket": lambda *a: bench_bucket(*a),
    "lsa_flat": lambda *a: bench_lsa(*a),
    "lsa_flat_threshold": lambda *a: bench_lsa(*a, threshold=True),
    "lsa_tree": lambda *a: bench_lsa_tree(*a),
    "lsa_tree_10m": lambda *a: bench_lsa_tree_levels(*a),
    "lsa_prefill_10m": lambda *a: bench_lsa(*a, threshold=True, workload="lsa_prefill_10m"),
    "lsa_prefill_10m_q4096": lambda *a: bench_lsa(*a, threshold=True, workload="lsa_prefill_10m_q4096"),
    "two_stage": lambda *a: bench_two_stage(*a),
    "two_stage_pq": lambda *a: bench_two_stage(*a, pq=True),
    "prefill_shard_merge": lambda *a: bench_shard_merge(*a),
    "attn_decode": lambda *a: bench_attention(*a),
}
# The lines a plain run times, each in a child process of its own: a fault in
# one (a sticky CUDA error ends its process) becomes an error entry and cannot
# reach the decode line or another variant.  A variant joins this list once it
# has run clean on a B200.
# the 4096-query LSA chunk is the scan's profile case, not a bench line
DEFAULT_VARIANTS = [v for v in VARIANTS if v != "lsa_prefill_10m_q4096"]


def bench_one_variant(L, args, peaks, peak_kind, name):
    """One variant in this process (``--only NAME``)."""
    return {name: VARIANTS[name](L, args, peaks, peak_kind)}


def bench_variants(args, names=None, timeout_s: float = 900.0):
    """Every variant in `names` in a child process of its own (``bench.py
    --only NAME``), one after another; each child's JSON line becomes that
    variant's entry, a child that fails leaves an error entry."""
    import subprocess
    res = {}
    for name in (DEFAULT_VARIANTS if names is None else names):
        cmd = [sys.executable, os.path.abspath(__file__), "--only", name, "--steps", str(args.steps),
               "--warmup", str(args.warmup)]
        env = dict(os.environ)
        for v in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "LOCAL_WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
            env.pop(v, None)
        t0 = time.perf_counter()
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=timeout_s, env=env, cwd=ROOT)
        except subprocess.TimeoutExpired:
            res[name] = {"error": f"timed out after {timeout_s:.0f} s"}
            continue
        entry = None
        for ln in reversed(r.stdout.splitlines()):
            if ln.startswith("{"):
                try:
                    entry = json.loads(ln).get(name)
                except ValueError:
                    entry = None
                break
        if r.returncode != 0 or not isinstance(entry, dict):
            tail = (r.stderr or r.stdout).strip().splitlines()[-3:]
            res[name] = {"error": f"exit {r.returncode}: " + " | ".join(tail)[-400:]}
        else:
            entry["child_wall_s"] = round(time.perf_counter() - t0, 1)
            res[name] = entry
    return res


def _profiled_loop(L, fn, steps, warm, st):
    """Warm up, time `steps` calls, then run them again with the library's
    per-kernel events on for the kernel breakdown (the step time is taken
    without the events, which add a few microseconds per launch)."""
    import torch
    for i in range(warm):
        fn(i, None)
    torch.cuda.synchronize()
    tot, _ = time_loop(fn, steps, 0, st)
    L.ls_profile_begin()
    time_loop(fn, steps, 0, st)
    prof = L.ls_profile_end()
    kern = {k: {"ms_per_step": v[0] / steps, "launches_per_step": v[1] / steps} for k, v in prof.items()}
    return tot / steps, kern


def _recall(sel, exact):
    """Mean over rows of |selected ∩ exact| / |exact| (padding -1 ignored)."""
    import torch
    hits, tot = 0, 0
    for r in range(sel.shape[0]):
        e = exact[r][exact[r] >= 0]
        a = sel[r][sel[r] >= 0]
        hits += int(torch.isin(a, e).sum())
        tot += int(e.numel())
    return hits / max(tot, 1)


def bench_prefill(L, args, peaks, peak_kind, full_scores=True, fp8=False):
    """Prefill chunk: history streamed from pinned host memory in 8192-key
    tiles through two device buffers, causal top-512 of 4096 queries; with
    fp8, e4m3 queries and an e4m3 history (the indexer's FP8 form)."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("prefill_chunk_fp8" if fp8 else "prefill_chunk")
    d = make_workload(wl)
    T, H, dd = d["q"].shape
    N = d["k"].shape[0]
    w, qp = to_dev(d["w"]), to_dev(d["q_pos"])
    out = (torch.empty((T, wl.k), dtype=torch.int32, device="cuda"),
           torch.empty((T, wl.k), dtype=torch.float32, device="cuda"))
    cs = torch.cuda.Stream()
    n_t = np.minimum((d["q_pos"] + 1) // wl.stride, N)
    pairs = int(n_t.sum())
    if fp8:
        q8, qs = to_dev(d["q8"]), to_dev(d["q_scale"])
        hk = torch.from_numpy(np.ascontiguousarray(d["k8"])).pin_memory()
        hs = torch.from_numpy(np.ascontiguousarray(d["k_scale"])).pin_memory()
        buf0 = torch.empty(wl.tile_keys * (dd + 4), dtype=torch.uint8, device="cuda")
        buf1 = torch.empty_like(buf0)
        ws = torch.empty(L.lib().ls_prefill_select_fp8_workspace_size(T, N, wl.tile_keys, wl.k, int(full_scores)),
                         dtype=torch.uint8, device="cuda")

        def pf(i, timed):
            L.ls_prefill_select_stream_fp8(q8, qs, w, qp, hk, hs, buf0, buf1, k=wl.k, stride=wl.stride,
                                           tile_keys=wl.tile_keys, full_scores=full_scores, ws=ws, out=out,
                                           copy_stream=cs)
            return None
        kname = "score_tc_kernel<8,fp8>"
    else:
        q = to_dev_bf16(d["q"])
        hist = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
        buf0 = torch.empty((wl.tile_keys, dd), dtype=torch.bfloat16, device="cuda")
        buf1 = torch.empty_like(buf0)
        ws = torch.empty(L.lib().ls_prefill_select_workspace_size(T, N, wl.tile_keys, wl.k, int(full_scores)),
                         dtype=torch.uint8, device="cuda")

        def pf(i, timed):
            L.ls_prefill_select_stream(q, w, qp, hist, buf0, buf1, k=wl.k, stride=wl.stride,
                                       tile_keys=wl.tile_keys, full_scores=full_scores, ws=ws, out=out,
                                       copy_stream=cs)
            return None
        kname = "score_tc_kernel<8>"

    ms, kern = _profiled_loop(L, pf, steps, warm, st)
    score_ms = kern[kname]["ms_per_step"]
    flops_alg = pairs * 2 * H * dd
    peak_t = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    if fp8:
        peak_t = 2 * peak_t   # fp8 dense = 2 x bf16 dense (4.5 vs 2.25 PFLOP/s nominal)
    res = {
        "ms_per_step": ms, "positions_per_s": pairs / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
        "kernels": kern,
        "roofline": roofline("tensor", flops_alg / (score_ms * 1e-3) / 1e12, peak_t, "TFLOP/s",
                             traffic=ncu_traffic(kname, wl.name if full_scores else wl.name + "_running"),
                             peak_kind=peak_kind + (" bf16 x 2 (fp8)" if fp8 else "")),
        "algorithmic_flops": flops_alg, "eligible_pairs": pairs,
        "workspace_bytes": ws.numel(),
        "note": ("step = 4 streamed 8192-key tiles (H2D on a copy stream) + causal top-512 of 4096 queries; "
                 + ("fp8 e4m3 queries and history (one scale per query head / per key); " if fp8 else "")
                 + ("full 4096 x 32768 score matrix, one top-k"
                    if full_scores else "running top-512 across tiles (first tile in full, later tiles filtered "
                                        "against each query's running 512th entry, merge per tile)")
                 + f"; roofline over the 4 scoring launches of the step ({kname})"),
    }
    del ws
    return res


def bench_bucket(L, args, peaks, peak_kind):
    """Bucket search over 32768 clusters of 8 keys, 256 queries."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("bucket")
    d = make_workload(wl)
    T, H, dd = d["q"].shape
    P_ = d["centroids"].shape[0]
    args_b = [to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev_bf16(d["centroids"]), to_dev(d["bucket_off"]),
              to_dev(d["bucket_mem"]), to_dev_bf16(d["keys"])]
    wsb = torch.empty(L.lib().ls_bucket_workspace_size(T, P_, wl.top_p, wl.budget), dtype=torch.uint8,
                      device="cuda")
    outb = (torch.empty((T, wl.k), dtype=torch.int32, device="cuda"),
            torch.empty((T, wl.k), dtype=torch.float32, device="cuda"))

    def bk(i, timed):
        L.ls_bucket_select(*args_b, top_p=wl.top_p, budget=wl.budget, k=wl.k, ws=wsb, out=outb)
        return None

    ms, kern = _profiled_loop(L, bk, steps, warm, st)
    cms = kern["score_tc_kernel<8>"]["ms_per_step"]
    # recall@k against the exact scan of every key (outside the timed region)
    N_ = d["keys"].shape[0]
    exact = L.ls_indexer_score(args_b[0].view(1, T, H, dd), args_b[1].view(1, T, H), args_b[5].view(1, N_, dd))
    ei, _ = L.ls_topk_select(exact.view(T, N_), wl.k)
    recall = _recall(outb[0], ei)
    del exact
    flops = T * P_ * 2 * H * dd
    peak_t = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    res = {"ms_per_step": ms, "positions_per_s": T * (P_ + wl.budget) / (ms * 1e-3),
           "selections_per_s": T / (ms * 1e-3), "kernels": kern,
           "roofline": roofline("tensor", flops / (cms * 1e-3) / 1e12, peak_t, "TFLOP/s",
                                traffic=ncu_traffic("score_tc_kernel<8>", wl.name), peak_kind=peak_kind),
           "algorithmic_flops_centroids": flops, "recall_at_k": recall,
           "note": "positions = centroids scored + keys rescored per query; roofline of the centroid scoring"}
    del args_b, wsb
    return res


def bench_lsa(L, args, peaks, peak_kind, threshold=False, workload="lsa_flat"):
    """Native LSA flat search: 256 index queries over 131072 buckets of one
    1048576-token sequence; top 1024 buckets, 4096 long-range keys.  With
    threshold, the sampled-threshold scan lists only the buckets that clear
    each query's threshold (else every score goes to a T x P matrix).  The
    prefill workload: 32768 queries over 1310720 buckets (threshold form
    only), a compute-bound scan reported against the bf16 tensor peak."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload(workload)
    d = make_workload(wl)
    ex = wl.extra
    T = d["q_idx"].shape[0]
    P_ = d["centroids"].shape[0]
    a = [to_dev_bf16(d["q_idx"]), to_dev(d["q_pos"]), to_dev_bf16(d["centroids"]), to_dev(d["bucket_off"]),
         to_dev(d["bucket_mem"])]
    ws = torch.empty(L.lib().ls_lsa_flat_workspace_size(T, P_, wl.top_p, int(threshold), 0), dtype=torch.uint8,
                     device="cuda")
    row = ex["n_sink"] + ex["block_keys"] + wl.budget
    out = (torch.empty((T, row), dtype=torch.int32, device="cuda"), torch.empty((T,), dtype=torch.int32, device="cuda"))

    def run(i, timed):
        L.ls_lsa_flat_select(*a, block_keys=ex["block_keys"], buckets_per_block=ex["bpb"], n_sink=ex["n_sink"],
                             top_p=wl.top_p, budget=wl.budget, threshold=threshold, ws=ws, out=out)
        return None

    ms, kern = _profiled_loop(L, run, steps, warm, st)
    kname = "dot_tc_kernel:filter" if threshold else "dot_tc_kernel"
    dms = kern[kname]["ms_per_step"]
    vis = np.minimum((d["q_pos"] // ex["block_keys"]) * ex["bpb"], P_)
    scored = int(vis.sum())
    # centroids and queries read; the full form also writes the T x P score matrix
    bytes_dot = P_ * 128 + T * 128 + (0 if threshold else T * P_ * 4)
    peak_b = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    traffic = ncu_traffic(kname, wl.name + ("_threshold" if threshold else ""))
    if T >= 4096:
        # prefill scale: the scan is a dense contraction (2 x 64 flops per visible (query, bucket) pair)
        rl = roofline("tensor", 128.0 * scored / (dms * 1e-3) / 1e12,
                      peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]), "TFLOP/s", traffic=traffic,
                      peak_kind=peak_kind)
    else:
        rl = roofline("hbm", bytes_dot / (dms * 1e-3) / 1e9, peak_b, "GB/s", traffic=traffic, peak_kind=peak_kind)
    res = {"ms_per_step": ms, "positions_per_s": scored / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
           "kernels": kern, "roofline": rl, "queries": T, "buckets": P_,
           "bytes_dot": bytes_dot, "visible_buckets_scored": scored,
           "note": "positions = visible buckets scored per query (one 64-d dot each); "
                   + ("sampled thresholds (every 128th bucket, 32nd best), the scan lists the buckets that clear "
                      "them, top-1024 of each list, full-scoring fallback launches that return at once; roofline "
                      "of the filtered scan over the centroid and query bytes it reads"
                      if threshold else "full T x P score matrix; roofline of the scoring over the centroids and "
                                        "queries read and the score matrix written")}
    del a, ws
    return res


def bench_lsa_tree(L, args, peaks, peak_kind):
    """LSA tree search on the lsa_flat sequence: 32768 node buckets scored,
    beam 2048, their 8192 child buckets scored, top 1024, read lists."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("lsa_tree")
    d = make_workload(wl)
    ex = wl.extra
    T = d["q_idx"].shape[0]
    P1 = d["node_centroids"].shape[0]
    a = [to_dev_bf16(d["q_idx"]), to_dev(d["q_pos"]), to_dev_bf16(d["centroids"]), to_dev_bf16(d["node_centroids"]),
         to_dev(d["bucket_off"]), to_dev(d["bucket_mem"])]
    ws = torch.empty(L.lib().ls_lsa_tree_workspace_size(T, P1, ex["beam"], ex["fanout"], ex["node_block"], wl.top_p),
                     dtype=torch.uint8, device="cuda")
    row = ex["n_sink"] + ex["block_keys"] + wl.budget
    out = (torch.empty((T, row), dtype=torch.int32, device="cuda"), torch.empty((T,), dtype=torch.int32, device="cuda"))

    def run(i, timed):
        L.ls_lsa_tree_select(*a, block_keys=ex["block_keys"], buckets_per_block=ex["bpb"], node_block=ex["node_block"],
                             fanout=ex["fanout"], beam=ex["beam"], n_sink=ex["n_sink"], top_p=wl.top_p,
                             budget=wl.budget, ws=ws, out=out)
        return None

    ms, kern = _profiled_loop(L, run, steps, warm, st)
    scored = T * (P1 + ex["beam"] * ex["fanout"])
    nms = kern["dot_tc_kernel:nodes"]["ms_per_step"]
    bytes_nodes = P1 * 128 + T * 128 + T * P1 * 4
    peak_b = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    res = {"ms_per_step": ms, "positions_per_s": scored / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
           "kernels": kern,
           "roofline": roofline("hbm", bytes_nodes / (nms * 1e-3) / 1e9, peak_b, "GB/s",
                                traffic=ncu_traffic("dot_tc_kernel", wl.name), peak_kind=peak_kind),
           "vectors_scored_per_query": P1 + ex["beam"] * ex["fanout"],
           "note": "positions = node buckets + child buckets scored per query (32768 + 8192 against 131072 for "
                   "the flat search); roofline of the node scoring (node centroids and queries read, scores "
                   "written)"}
    del a, ws
    return res


def bench_lsa_tree_levels(L, args, peaks, peak_kind, workload="lsa_tree_10m"):
    """LSA tree search over three node levels at 10485760 tokens: 256 index
    queries; the beam starts at level 3 (20480 node buckets), keeps 2048,
    steps down through levels 2 and 1 to the buckets, top 1024, read lists."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload(workload)
    d = make_workload(wl)
    ex = wl.extra
    T = d["q_idx"].shape[0]
    P_ = d["centroids"].shape[0]
    levels = [to_dev_bf16(x) for x in d["node_levels"]]
    sizes = [x.shape[0] for x in d["node_levels"]]
    a = [to_dev_bf16(d["q_idx"]), to_dev(d["q_pos"]), to_dev_bf16(d["centroids"]), levels, to_dev(d["bucket_off"]),
         to_dev(d["bucket_mem"])]
    kw = dict(node_block=ex["node_block"], fanout=ex["fanout"], beam=ex["beam"], start_nodes=ex["start_nodes"],
              top_p=wl.top_p)
    ws = torch.empty(L.ls_lsa_tree_levels_workspace_size(T, P_, sizes, **kw), dtype=torch.uint8, device="cuda")
    row = ex["n_sink"] + ex["block_keys"] + wl.budget
    out = (torch.empty((T, row), dtype=torch.int32, device="cuda"), torch.empty((T,), dtype=torch.int32, device="cuda"))

    def run(i, timed):
        L.ls_lsa_tree_levels_select(*a, block_keys=ex["block_keys"], buckets_per_block=ex["bpb"],
                                    n_sink=ex["n_sink"], budget=wl.budget, ws=ws, out=out, **kw)
        return None

    ms, kern = _profiled_loop(L, run, steps, warm, st)
    # vectors scored per query: the start level's visible nodes, then the beam's children (and any
    # uncovered entries) at each level below, from the level sizes the oracle's visibility rule gives
    start = next((i + 1 for i, n in enumerate(sizes) if n <= ex["start_nodes"]), len(sizes))
    vis0 = np.minimum((d["q_pos"] // ex["block_keys"]) * ex["bpb"], P_)
    per_query, cand_rows = [], 0
    for v0 in vis0:
        v = [int(v0)]
        for n in sizes:
            v.append(min(n, v[-1] // ex["node_block"] * (ex["node_block"] // ex["fanout"])))
        below = sum(min(ex["beam"], v[lv + 1]) * ex["fanout"] + (v[lv] - ex["fanout"] * v[lv + 1])
                    for lv in range(start - 1, -1, -1))
        per_query.append(v[start] + below)
        cand_rows += below
    scored = int(np.sum(per_query))
    cand_ms = kern["lsa_tree_candidates_kernel"]["ms_per_step"]
    peak_b = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    res = {"ms_per_step": ms, "positions_per_s": scored / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
           "kernels": kern, "start_level": start, "level_sizes": [P_] + sizes,
           "vectors_scored_per_query": float(np.mean(per_query)), "flat_vectors_per_query": float(np.mean(vis0)),
           "roofline": roofline("hbm", cand_rows * 136 / (cand_ms * 1e-3) / 1e9, peak_b, "GB/s", peak_kind=peak_kind),
           "note": "positions = vectors scored per query (start-level nodes, then each level's candidates), "
                   "summed; roofline of the candidate scoring below the start level (136 bytes per candidate: "
                   "its 128-byte centroid gathered, score and label written); inputs 168 MB of bucket centroids "
                   "(larger than L2) of which each step gathers a part; no flush"}
    del a, ws, levels
    return res


def bench_shard_merge(L, args, peaks, peak_kind, shards: int = 4):
    """Combine step of a history-sharded prefill: the prefill chunk's history
    in 4 contiguous shards, each shard's top-512 lists computed once outside
    the timed region, then ls_merge_select (pack the valid prefixes with the
    shards' first positions, exact top-512 of 4 x 512 candidates per query)
    timed per step."""
    import torch
    from sparse_attention_indexer_lightning_b200 import shard_plan
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("prefill_chunk")
    d = make_workload(wl)
    T = d["q"].shape[0]
    N = d["k"].shape[0]
    q, w, qp = to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev(d["q_pos"])
    vals, idxs, offs = [], [], []
    for base, length in shard_plan(N, shards):
        hist = torch.from_numpy(np.ascontiguousarray(d["k"][base:base + length]).view(np.int16)).view(
            torch.bfloat16).pin_memory()
        buf0 = torch.empty((wl.tile_keys, 128), dtype=torch.bfloat16, device="cuda")
        buf1 = torch.empty_like(buf0)
        i_s, v_s = L.ls_prefill_select_stream(q, w, qp - base * wl.stride, hist, buf0, buf1, k=wl.k,
                                              stride=wl.stride, tile_keys=wl.tile_keys)
        vals.append(v_s)
        idxs.append(i_s)
        offs.append(base)
    vals, idxs = torch.stack(vals), torch.stack(idxs)
    offs = to_dev(np.asarray(offs, dtype=np.int32))
    ws = torch.empty(L.lib().ls_merge_select_workspace_size(shards, T, wl.k), dtype=torch.uint8, device="cuda")
    out = (torch.empty((T, wl.k), dtype=torch.int32, device="cuda"),
           torch.empty((T, wl.k), dtype=torch.float32, device="cuda"))

    def run(i, timed):
        L.ls_merge_select(vals, idxs, offs, k=wl.k, ws=ws, out=out)
        return None

    ms, kern = _profiled_loop(L, run, steps, warm, st)
    tk = kern["topk_kernel"]["ms_per_step"]
    cand = shards * T * wl.k
    peak_b = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    res = {"ms_per_step": ms, "selections_per_s": T / (ms * 1e-3), "candidates_per_s": cand / (ms * 1e-3),
           "kernels": kern,
           "roofline": roofline("hbm", (cand * 8 + T * wl.k * 8) / (tk * 1e-3) / 1e9, peak_b, "GB/s",
                                peak_kind=peak_kind),
           "note": "top-k of the packed candidates: 8 bytes per candidate read (value, position) and 8 per "
                   "selected entry written; the shards' own selections are outside the timed region"}
    del vals, idxs, ws, out
    return res


# fp32 FMA issue rate of the CUDA cores: 148 SMs x 128 lanes x 2 flops x 1.965 GHz (clocks.max.sm)
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bench_attention(L, args, peaks, peak_kind):
    """Sparse main attention after the decode selection: 64 queries x 128
    heads, each over its 512 selected rows of a 262144 x 576 bf16 latent cache
    (302 MB).  Four selections are cycled so that consecutive steps gather
    different rows (4 x 37.7 MB, more than L2)."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("attn_decode")
    d = make_workload(wl)
    T, H, D = d["q"].shape
    R = d["latent"].shape[0]
    rng = np.random.default_rng(wl.seed + 1)
    sets = [to_dev(d["idx"])] + [to_dev(np.stack([rng.choice(R, size=wl.k, replace=False) for _ in range(T)])
                                        .astype(np.int32)) for _ in range(3)]
    q, lat = to_dev_bf16(d["q"]), to_dev_bf16(d["latent"])
    out = torch.empty((T, H, 512), dtype=torch.float32, device="cuda")

    def run(i, timed):
        L.ls_sparse_attention(q, lat, sets[i % len(sets)], out=out)
        return None

    def run_cc(i, timed):
        L.ls_sparse_attention(q, lat, sets[i % len(sets)], out=out, cuda_cores=True)
        return None

    ms, kern = _profiled_loop(L, run, steps, warm, st)
    kname = "sparse_attn_tc_kernel" if "sparse_attn_tc_kernel" in kern else "sparse_attn_kernel"
    kms = kern[kname]["ms_per_step"]
    ms_cc, kern_cc = _profiled_loop(L, run_cc, steps, warm, st)
    flops = T * H * wl.k * (D + 512) * 2
    gathered = T * wl.k * D * 2
    peak_b = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    peak_t = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    res = {"ms_per_step": ms, "positions_per_s": T * wl.k / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
           "kernels": kern,
           "roofline": roofline("tensor", flops / (kms * 1e-3) / 1e12, peak_t, "TFLOP/s",
                                traffic=ncu_traffic("sparse_attn_tc_kernel", wl.name), peak_kind=peak_kind),
           "gather_hbm_frac": round(gathered / (kms * 1e-3) / 1e9 / peak_b, 4),
           "cuda_core_kernel": {"ms_per_step": ms_cc, "kernels": kern_cc,
                                "alu_frac": round(flops / (kern_cc["sparse_attn_kernel"]["ms_per_step"] * 1e-3)
                                                  / 1e12 / ALU_FP32_TFLOPS, 4)},
           "note": "positions = selected rows attended per step; flops = T x H x k x (576 + 512) x 2 (logits and "
                   "values, counted once; the tensor-core kernel computes the logits in both CTAs of a query); "
                   "tensor-core kernel (bf16 weights in the value contraction), the fp32 CUDA-core kernel timed "
                   "beside it on the same selections"}
    del sets, q, lat, out
    return res


def bench_two_stage(L, args, peaks, peak_kind, pq=False):
    """Two-stage decode search: compact scan (int8 + scale, or 32-byte PQ codes), shortlist, exact re-rank."""
    import torch
    from workloads import get_workload, make_workload
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)
    wl = get_workload("two_stage_pq" if pq else "two_stage")
    d = make_workload(wl)
    B, H, dd = d["q"].shape
    N = d["fk"].shape[1]
    fk = [to_dev(d["fk"]).view(torch.float8_e4m3fn), to_dev(d["fk_scale"])]
    if pq:
        books = torch.from_numpy(d["pq_books"].view(np.int16)).view(torch.float16).cuda()
        a2 = [to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev(d["pq_codes"]), books] + fk
        call = L.ls_decode_two_stage_pq_select
        scan_name, scan_bytes = "score_q8_kernel<pq>", B * N * 32
    else:
        a2 = [to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev(d["ck"]), to_dev(d["ck_scale"])] + fk
        call = L.ls_decode_two_stage_select
        scan_name, scan_bytes = "score_q8_kernel<int8>", B * N * (dd + 4)
    ws2 = torch.empty(L.lib().ls_two_stage_workspace_size(B, N, wl.shortlist), dtype=torch.uint8, device="cuda")
    out2 = (torch.empty((B, wl.k), dtype=torch.int32, device="cuda"),
            torch.empty((B, wl.k), dtype=torch.float32, device="cuda"))

    def ts(i, timed):
        call(*a2, shortlist=wl.shortlist, k=wl.k, ws=ws2, out=out2)
        return None

    ms, kern = _profiled_loop(L, ts, steps, warm, st)
    scan_ms = kern[scan_name]["ms_per_step"]
    # recall@k against the exact full scan of the fp8 keys (outside the timed region)
    nv = to_dev(d["n_valid"]) if d.get("n_valid") is not None else None
    exact = L.ls_indexer_score(a2[0].view(B, 1, H, dd), a2[1].view(B, 1, H), fk[0], key_scale=fk[1], n_valid=nv)
    ei, _ = L.ls_topk_select(exact.view(B, N), wl.k, n_valid=nv)
    recall = _recall(out2[0], ei)
    del exact
    res = {
        "ms_per_step": ms, "positions_per_s": B * (N + wl.shortlist) / (ms * 1e-3),
        "selections_per_s": B / (ms * 1e-3), "kernels": kern,
        "roofline": roofline("hbm", scan_bytes / (scan_ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                             traffic=ncu_traffic(scan_name, wl.name), peak_kind=peak_kind),
        "algorithmic_bytes_scan": scan_bytes, "recall_at_k": recall,
        "note": "positions = compact keys scanned + shortlist re-ranked; roofline of the compact scan "
                + ("(32-byte PQ codes; codebooks stay in shared memory)" if pq else "(int8 codes + fp32 scales)"),
    }
    del a2, ws2
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- #
# CPU oracle legs
# --------------------------------------------------------------------------- #
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [x.get("num_threads", 1) for x in info if x.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_decode_rate(d, budget_s: float, k: int):
    """Oracle decode selection over whole sequences (cycling through the
    batch) until budget_s of CPU time has elapsed."""
    from oracle.select import decode_select
    B, N = d["k"].shape[0], d["k"].shape[1]
    done = 0
    t0 = time.perf_counter()
    while (time.perf_counter() - t0) < budget_s:
        b = done % B
        decode_select(d["q"][b:b + 1], d["w"][b:b + 1], d["k"][b:b + 1], None, k)
        done += 1
    el = time.perf_counter() - t0
    return done * N / el, done, el


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import get_workload, make_workload
    wl = get_workload(args.workload)
    d = make_workload(wl)
    B, N = d["k"].shape[0], d["k"].shape[1]
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_decode_rate(d, per_step_budget / 4, wl.k)
    rates, seqs = [], 0
    for _ in range(args.steps):
        r, n, _ = oracle_decode_rate(d, per_step_budget, wl.k)
        rates.append(r)
        seqs += n
    value = statistics.median(rates)
    cores = blas_threads()
    H, dd = d["q"].shape[1], d["q"].shape[2]
    line = {
        "impl": "reference", "metric": "indexer query-positions scored/sec (decode selection, top-512)",
        "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # the time one step of the workload (all B sequences) takes at the measured rate
        "ms_per_step": B * N / value * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": decode_config(wl, B, N, H, dd, 1),
        "cpu_baseline": {"value": value, "unit": "positions/s", "cores": cores, "kind": "oracle",
                         "sample": f"whole sequences of {N} positions cycled through the batch for about "
                                   f"{per_step_budget:.0f} s per timed step, {seqs} in total over {args.steps} "
                                   f"steps; value = the median step's rate, ms_per_step = a {B}-sequence step "
                                   f"at that rate"},
        "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- #
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 200 decode steps (about 23 ms of timed work) give the clock sampler a
    # dozen or more NVML readings inside the timed region
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_batch")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--variants", default="default",
                    help="'default' (the lines that have run clean on a B200), 'all', or a comma-separated list")
    ap.add_argument("--only", default=None, choices=sorted(VARIANTS),
                    help="time one variant in this process and skip the decode line (profiling, and the "
                         "child processes of a plain run)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world, rank, local = dist_setup(args.gpus)
    import sparse_attention_indexer_lightning_b200 as L
    peaks, peak_kind = load_peaks()
    if args.only:
        print(json.dumps({"variant": args.only, **bench_one_variant(L, args, peaks, peak_kind, args.only)}))
        return 0
    out, d = bench_decode(L, args, world, rank, peaks, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n_seq, el = oracle_decode_rate(d, 12.0, 512)
        out["cpu_baseline"] = {"value": rate, "unit": "positions/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{n_seq} whole sequences x {d['k'].shape[1]} positions "
                                         f"({el:.1f} s of fp64 oracle work)"}
    del d
    if not args.no_variants and world == 1:
        names = (None if args.variants == "default" else sorted(VARIANTS) if args.variants == "all"
                 else [v for v in args.variants.split(",") if v])
        try:
            out["variants"] = bench_variants(args, names)
        except Exception as e:  # noqa: BLE001 -- the decode line is printed whatever happens here
            out["variants"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
