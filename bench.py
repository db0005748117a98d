"""Benchmark of the lightning-indexer selection path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_batch] [--no-variants] [--no-cpu-baseline]

One step is one decode selection over the batch workload: 64 sequences x
32768 stride-4 compressed bf16 keys (131072 tokens each), 32 heads x 128 dims,
exact top-512 per sequence -- the scan (ls_indexer_score) then the selection
(ls_topk_select).  Inputs (537 MB of keys) are larger than the 126 MB L2, so
no flush is needed between steps.  The metric is query-positions scored per
second (selections per second alongside).  The prefill, two-stage and bucket
searches are timed the same way and reported under "variants", each with the
roofline of its dominant kernel.

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
import subprocess
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
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- #
# distributed plumbing
# --------------------------------------------------------------------------- #
def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


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
    sc = torch.empty((B, 1, N), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, wl.k), dtype=torch.int32, device="cuda")
    val = torch.empty((B, wl.k), dtype=torch.float32, device="cuda")
    lib = L.lib()
    import ctypes
    P = ctypes.c_void_p
    stp = P(st.cuda_stream)

    def step(i, timed):
        e0 = e1 = e2 = None
        if timed:
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(st)
        s1 = lib.ls_indexer_score(P(q4.data_ptr()), P(w3.data_ptr()), P(k.data_ptr()), 0, None, None, None, 4,
                                  B, 1, H, dd, N, P(sc.data_ptr()), stp)
        if timed:
            e1.record(st)
        s2 = lib.ls_topk_select(P(sc.data_ptr()), N, None, B, N, wl.k, P(idx.data_ptr()), P(val.data_ptr()), stp)
        if s1 or s2:
            raise RuntimeError(lib.ls_last_error().decode())
        if timed:
            e2.record(st)
            return {"scan": (e0, e1), "topk": (e1, e2)}
        return None

    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    total_ms, seg = time_loop(step, args.steps, args.warmup, st)
    clk = clocks.stop()
    barrier(world)
    ms_per_step = max_over_ranks(total_ms / args.steps, world)
    scan_ms = seg["scan"] / args.steps
    positions = B * N
    value = world * positions / (ms_per_step * 1e-3)
    key_bytes = B * N * dd * 2
    out = {
        "metric": "indexer query-positions scored/sec (decode selection, top-512)",
        "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(d) keys and queries, N(0,1)/sqrt(H) head weights)",
        "config": {"workload": wl.name, "sequences_per_gpu": B, "compressed_positions": N, "tokens_per_sequence": 4 * N,
                   "heads": H, "d": dd, "k": wl.k, "parallelism": f"replicas x{world}",
                   "l2": "inputs (537 MB keys) larger than the 126 MB L2; no flush"},
        "selections_per_s": world * B / (ms_per_step * 1e-3),
        "breakdown_ms": {"scan": scan_ms, "topk": seg["topk"] / args.steps},
        "roofline": roofline("hbm", key_bytes / (scan_ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                             traffic=args.scan_traffic, peak_kind=peak_kind),
        "gpu_launches": 2 * args.steps,
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
    ws = torch.empty(lib.ls_decode_select_workspace_size(B, N), dtype=torch.uint8, device="cuda")

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


def bench_variants(L, args, peaks, peak_kind):
    """Prefill chunk, two-stage and bucket searches: one timed loop each."""
    import torch
    from workloads import get_workload, make_workload
    res = {}
    st = torch.cuda.current_stream()
    steps = max(3, args.steps)
    warm = max(3, args.warmup)

    # ---- prefill chunk: streamed history, causal top-512 --------------------
    wl = get_workload("prefill_chunk")
    d = make_workload(wl)
    T, H, dd = d["q"].shape
    N = d["k"].shape[0]
    q, w, qp = to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev(d["q_pos"])
    hist = torch.from_numpy(d["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hist_dev = hist.cuda()
    buf0 = torch.empty((wl.tile_keys, dd), dtype=torch.bfloat16, device="cuda")
    buf1 = torch.empty_like(buf0)
    ws = torch.empty(L.lib().ls_prefill_select_workspace_size(T, N), dtype=torch.uint8, device="cuda")
    out = (torch.empty((T, wl.k), dtype=torch.int32, device="cuda"),
           torch.empty((T, wl.k), dtype=torch.float32, device="cuda"))
    cs = torch.cuda.Stream()
    n_t = np.minimum((d["q_pos"] + 1) // wl.stride, N)
    pairs = int(n_t.sum())

    def pf(i, timed, src):
        L.ls_prefill_select_stream(q, w, qp, src, buf0, buf1, k=wl.k, stride=wl.stride, tile_keys=wl.tile_keys,
                                   ws=ws, out=out, copy_stream=cs)
        return None

    tot, _ = time_loop(lambda i, t: pf(i, t, hist), steps, warm, st)
    ms = tot / steps
    # scoring kernels alone: the same 4 tile launches over device-resident history
    sc = torch.empty((1, T, N), dtype=torch.float32, device="cuda")
    lib = L.lib()
    import ctypes
    P = ctypes.c_void_p

    def score_only(i, timed):
        e0 = e1 = None
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
        s = lib.ls_indexer_score(P(q.data_ptr()), P(w.data_ptr()), P(hist_dev.data_ptr()), 0, None, None,
                                 P(qp.data_ptr()), wl.stride, 1, T, H, dd, N, P(sc.data_ptr()), P(st.cuda_stream))
        if s:
            raise RuntimeError(lib.ls_last_error().decode())
        if timed:
            e1.record(st)
            return {"score": (e0, e1)}
        return None

    _, seg = time_loop(score_only, steps, warm, st)
    score_ms = seg["score"] / steps
    flops_alg = pairs * 2 * H * dd
    peak_t = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    res["prefill_chunk"] = {
        "ms_per_step": ms, "positions_per_s": pairs / (ms * 1e-3), "selections_per_s": T / (ms * 1e-3),
        "score_kernel_ms": score_ms,
        "roofline": roofline("tensor", flops_alg / (score_ms * 1e-3) / 1e12, peak_t, "TFLOP/s", peak_kind=peak_kind),
        "algorithmic_flops": flops_alg, "eligible_pairs": pairs,
        "note": "step = 4 streamed 8192-key tiles (H2D on a copy stream) + causal top-512 of 4096 queries; "
                "score_kernel_ms = scoring of the whole history resident in HBM (one launch)",
    }
    del sc, ws, hist_dev

    # ---- bucket search -------------------------------------------------------
    wl = get_workload("bucket")
    d = make_workload(wl)
    T = d["q"].shape[0]
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

    tot, _ = time_loop(bk, steps, warm, st)
    ms = tot / steps
    res["bucket"] = {"ms_per_step": ms, "positions_per_s": T * (P_ + wl.budget) / (ms * 1e-3),
                     "selections_per_s": T / (ms * 1e-3),
                     "note": "positions = centroids scored + keys rescored per query"}
    del args_b, wsb

    # ---- two-stage decode search ---------------------------------------------
    wl = get_workload("two_stage")
    d = make_workload(wl)
    B, H, dd = d["q"].shape
    N = d["ck"].shape[1]
    a2 = [to_dev_bf16(d["q"]), to_dev(d["w"]), to_dev(d["ck"]), to_dev(d["ck_scale"]),
          to_dev(d["fk"]).view(torch.float8_e4m3fn), to_dev(d["fk_scale"])]
    ws2 = torch.empty(L.lib().ls_two_stage_workspace_size(B, N, wl.shortlist), dtype=torch.uint8, device="cuda")
    out2 = (torch.empty((B, wl.k), dtype=torch.int32, device="cuda"),
            torch.empty((B, wl.k), dtype=torch.float32, device="cuda"))

    def ts(i, timed):
        L.ls_decode_two_stage_select(*a2, shortlist=wl.shortlist, k=wl.k, ws=ws2, out=out2)
        return None

    tot, _ = time_loop(ts, steps, warm, st)
    ms = tot / steps
    # the compact scan alone
    s_hat = torch.empty((B, 1, N), dtype=torch.float32, device="cuda")

    def scan_only(i, timed):
        e0 = e1 = None
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
        L.ls_indexer_score(a2[0].view(B, 1, H, dd), a2[1].view(B, 1, H), a2[2], key_scale=a2[3])
        if timed:
            e1.record(st)
            return {"scan": (e0, e1)}
        return None

    _, seg = time_loop(scan_only, steps, warm, st)
    scan_ms = seg["scan"] / steps
    scan_bytes = B * N * (dd + 4)
    res["two_stage"] = {
        "ms_per_step": ms, "positions_per_s": B * (N + wl.shortlist) / (ms * 1e-3),
        "selections_per_s": B / (ms * 1e-3), "compact_scan_ms": scan_ms,
        "roofline": roofline("hbm", scan_bytes / (scan_ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s",
                             peak_kind=peak_kind),
        "algorithmic_bytes_scan": scan_bytes,
        "note": "positions = compact keys scanned + shortlist re-ranked; scan roofline on int8 codes + scales",
    }
    del a2, ws2, s_hat
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
    """Oracle decode selection over whole sequences until budget_s elapses."""
    from oracle.select import decode_select
    B, N = d["k"].shape[0], d["k"].shape[1]
    done = 0
    t0 = time.perf_counter()
    while done < B and (time.perf_counter() - t0) < budget_s:
        decode_select(d["q"][done:done + 1], d["w"][done:done + 1], d["k"][done:done + 1], None, k)
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
    line = {
        "impl": "reference", "metric": "indexer query-positions scored/sec (decode selection, top-512)",
        "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": N / value * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": {"workload": wl.name, "sequences": B, "compressed_positions": N},
        "cpu_baseline": {"value": value, "unit": "positions/s", "cores": cores, "kind": "oracle",
                         "sample": f"whole sequences of {N} positions, {seqs} in total over {args.steps} steps"},
        "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- #
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_batch")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scan-traffic", type=float, default=None,
                    help="dram bytes per scan launch from an ncu capture of the current kernel")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world, rank, local = dist_setup(args.gpus)
    import sparse_attention_indexer_lightning_b200 as L
    peaks, peak_kind = load_peaks()
    out, d = bench_decode(L, args, world, rank, peaks, peak_kind)
    if not args.no_variants and world == 1:
        out["variants"] = bench_variants(L, args, peaks, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n_seq, el = oracle_decode_rate(d, 15.0, 512)
        out["cpu_baseline"] = {"value": rate, "unit": "positions/s", "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{n_seq} whole sequences x {d['k'].shape[1]} positions "
                                         f"({el:.1f} s of fp64 oracle work)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
