"""Benchmark of the ALHR inference path: routed queries per second on one step of the
configured workload (tree build + fused route/attend over every query), on N GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl alhr|reference]

N > 1 runs one process per GPU under torch.distributed.run (weak scaling: every rank processes
its own full workload with its own seed; no collective on the data path). Prints one JSON line
on rank 0. Inputs are seeded synthetic tensors generated on the device; L2 is flushed by a
512 MiB write before every timed step; the timed region holds exactly K steps bracketed by a
barrier and a device synchronisation; each step is timed with CUDA events on the launch stream
and the job time is the maximum over ranks.

--impl reference times the oracle (the plain CPU reference that the tests use) on the host
cores, on a bounded sample of the same workload, with the same metric.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "routed queries/sec and achieved HBM GB/s vs ~8 TB/s roofline, N=16384, 1 B200"
DEFAULT_WORKLOAD = "prefill_b2h8_n16384"
L2_FLUSH_BYTES = 512 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="alhr", choices=["alhr", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--labels", action="store_true",
                    help="instead of the bench line: time the phase-2 label kernel "
                         "(alhr_topk_labels, top-16 keys of every query) on the workload (1 GPU)")
    ap.add_argument("--stages", action="store_true",
                    help="instead of the bench line: per-stage times of the workload through the "
                         "unfused entry points, and fused-forward time against N (1 GPU)")
    ap.add_argument("--launch-mode", default="auto", choices=["auto", "throughput", "latency"],
                    help="with --stages: launch shape of the per-query kernels")
    ap.add_argument("--no-sweep", action="store_true",
                    help="with --stages: only the workload's own stage split (no sweep over N)")
    ap.add_argument("--tree", action="store_true",
                    help="instead of the bench line: time the tree build (alhr_build_tree) on "
                         "the workload's keys (1 GPU)")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --tree: replace the workload's batch (sequences)")
    ap.add_argument("--cpu-sample-stride", type=int, default=4,
                    help="CPU baseline: every k-th query row of every (b,h) block")
    ap.add_argument("--ref-stride", type=int, default=64,
                    help="--impl reference: every k-th query row of each step's block")
    return ap.parse_args()


def describe(wl) -> str:
    pred = (f"predictor W int8 U[{wl.w_lo},{wl.w_hi}] 32x{2 * wl.d}" if wl.predictor
            else f"fixed budget min(i+1,{wl.fixed_budget_cap})")
    extra = f", {wl.plant_pairs} planted pairs/seq" if wl.plant_pairs else ""
    return (f"{wl.name}: batch {wl.batch}, heads {wl.heads}, N={wl.n}, d={wl.d}, "
            f"queries [{wl.q_start},{wl.q_start + wl.nq}), w={wl.window}, max_keys={wl.max_keys}, "
            f"Q/K int8 U[{wl.qk_lo},{wl.qk_hi}], V bf16 N(0,1), {pred}{extra}")


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), world
    return None, 0, 1


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float) -> float:
    """The largest x over all ranks (NCCL on the GPU, gloo on the host)."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle (CPU) timing

def oracle_sample(wl, stride: int, blocks=None, inp=None) -> dict:
    """The oracle as it stands, on the host cores, on a bounded sample of the workload: for
    each listed (b,h) block, its whole tree and every `stride`-th query row. Blocks run on a
    thread pool, one block per thread (the oracle itself is single-threaded; ctypes releases
    the GIL). The sample's wall time is scaled to all query rows of the listed blocks, and
    the value is queries of those blocks per extrapolated second."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as orc
    from tree_routed_sparse_b200 import synth

    orc.lib()
    if inp is None:
        inp = synth.make_inputs(wl, "cpu")
    if blocks is None:
        blocks = [(b, h) for b in range(wl.batch) for h in range(wl.heads)]
    rows = np.arange(0, wl.nq, max(1, min(stride, wl.nq)), dtype=np.int32)
    Vbits = inp["V"].view(torch.int16).numpy().view(np.uint16)
    W = None if inp["W"] is None else inp["W"].numpy()

    def run(bh):
        b, h = bh
        K = inp["K"][b, h].numpy()
        Q = inp["Q"][b, h].numpy()
        bo = None if inp["budget_override"] is None else inp["budget_override"][b, h].numpy()
        t0 = time.perf_counter()
        nodes = orc.build_tree(K)
        t1 = time.perf_counter()
        orc.forward(Q, K, Vbits[b, h], nodes, W, bo, q_start=wl.q_start, window=wl.window,
                    max_keys=wl.max_keys, rows=rows)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1

    threads = max(1, min(os.cpu_count() or 1, len(blocks)))
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(run, blocks))
    wall = time.perf_counter() - t0
    t_tree = sum(r[0] for r in res)
    t_route = sum(r[1] for r in res)
    scale = wl.nq / len(rows)
    est_wall = wall * (t_tree + t_route * scale) / (t_tree + t_route)
    total_q = len(blocks) * wl.nq
    return {"value": total_q / est_wall, "unit": "queries/s", "cores": threads,
            "kind": "oracle",
            "sample": (f"{describe(wl)}; {len(blocks)} (b,h) blocks: each whole tree plus "
                       f"every {max(1, min(stride, wl.nq))}-th query row ({len(rows)} of "
                       f"{wl.nq}), time scaled to all rows; {threads} threads, one block per "
                       f"thread; sample wall {wall:.2f} s"),
            "sample_wall_s": wall}


# ------------------------------------------------------------------ the GPU arm

def run_alhr(args, dist, rank, world):
    from tree_routed_sparse_b200 import alhr, metrics, synth
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.WORKLOADS[args.workload].replace(seed=synth.WORKLOADS[args.workload].seed + rank)
    vb = max(-wl.qk_lo, wl.qk_hi)
    inp = synth.make_inputs(wl, dev)
    Q, K, V, W, bo = inp["Q"], inp["K"], inp["V"], inp["W"], inp["budget_override"]
    tree = torch.empty((wl.batch, wl.heads, alhr.tree_bytes(wl.n, wl.d, vb)), dtype=torch.uint8,
                       device=dev)
    out = torch.empty((wl.batch, wl.heads, wl.nq, wl.d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits, value_bound=vb)

    def step():
        alhr.build_tree(K, tree, value_bound=vb)
        alhr.forward(Q, K, V, tree, W=W, budget_override=bo, out=out, **kw)

    # one untimed run with every output: counts for the byte model
    alhr.build_tree(K, tree, value_bound=vb)
    full = alhr.forward(Q, K, V, tree, W=W, budget_override=bo, want_count=True,
                        want_expansions=True, want_budget=True, **kw)
    torch.cuda.synchronize()
    pos = np.broadcast_to(np.arange(wl.q_start, wl.q_start + wl.nq), (wl.bh, wl.nq))
    fwd_bytes = metrics.forward_bytes(pos, wl.n, wl.d, wl.window, full["count"].cpu().numpy(),
                                      full["expansions"].cpu().numpy(),
                                      full["budget"].cpu().numpy(), wl.predictor, wl.max_keys,
                                      value_bound=vb)
    tree_bytes = metrics.tree_bytes(wl.bh, wl.n, wl.d, vb)
    mean_keys = float(full["count"].float().mean())
    mean_budget = float(full["budget"].float().mean())
    del full

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(dist)
    torch.cuda.synchronize()
    sampler.start()
    wall0 = time.perf_counter()
    for s in range(args.steps):
        flush.fill_(s & 0xFF)
        ev[s][0].record(stream)
        alhr.build_tree(K, tree, value_bound=vb)
        ev[s][1].record(stream)
        alhr.forward(Q, K, V, tree, W=W, budget_override=bo, out=out, **kw)
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(dist)
    clocks = sampler.stop()
    t_tree = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_fwd = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_step = t_tree + t_fwd
    t_job = max_over_ranks(dist, t_step)
    queries = wl.bh * wl.nq
    value = world * queries * args.steps / t_job

    # end to end through the public API, host buffers: every step copies its inputs in from
    # pinned memory, builds the tree, runs the fused forward and copies the output back, through
    # tree_routed_sparse_b200.pipeline.HostPipeline (copies of the next and the previous step
    # overlap this step's kernels on their own streams; L2 flushed on the compute stream before
    # every step, inside the timed region)
    from tree_routed_sparse_b200.pipeline import HostPipeline
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in inp.items()}
    outs_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    pipe = HostPipeline(host, device=dev, flush=flush, **kw)
    for s in range(3):
        pipe.submit(host, outs_host[s & 1])
    pipe.synchronize()
    assert torch.equal(outs_host[0], out.cpu()) and torch.equal(outs_host[1], out.cpu())
    barrier(dist)
    torch.cuda.synchronize()
    e2e_start, e2e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_start.record(pipe.copy_in)
    for s in range(args.e2e_steps):
        pipe.submit(host, outs_host[s & 1])
    e2e_end.record(pipe.copy_out)
    pipe.synchronize()
    barrier(dist)
    t_e2e = max_over_ranks(dist, e2e_start.elapsed_time(e2e_end) / 1e3)
    e2e_value = world * queries * args.e2e_steps / t_e2e

    if rank != 0:
        return None

    peaks = {}
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    fwd_launch_s = t_fwd / args.steps
    achieved = fwd_bytes / fwd_launch_s / 1e9
    rec = profiled_record(args.workload)
    traffic = rec.get("dram_bytes_per_launch") if rec else None
    tree_launches = tree_build_launches(wl.bh, wl.n)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "queries/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_job / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int32",
        "data": "synthetic (seeded SplitMix64; random int8 predictor weights, no trained model)",
        "config": {
            "workload": describe(wl),
            "queries_per_step_per_gpu": queries,
            "step": "alhr_build_tree + alhr_forward (fused budget, window, descent, attention)",
            "l2": "flushed by a 512 MiB write before every timed step (not timed)",
            "parallelism": f"{world} independent replica(s), one per GPU, no collective",
            "score_bits": 32 if alhr.score_bits(alhr.make_dims(Q, K, **kw)) == 32 else 64,
            "mean_keys_per_query": mean_keys,
            "mean_budget": mean_budget,
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "query_kernel (fused alhr_forward)",
            "achieved": achieved,
            "peak": peak,
            "unit": "GB/s",
            "frac": achieved / peak,
            "peak_source": f"{peak_src} hbm_gbs",
            "algorithmic_bytes_per_launch": fwd_bytes,
            "launch_ms": fwd_launch_s * 1e3,
            "traffic": traffic,
            "issue": issue_rate(rec, fwd_launch_s),
            "note": ("algorithmic bytes count every row the path reads as if from DRAM; "
                     "queries run in (b, h, i) order, so the rows in use at any time (about "
                     "one head's tree, keys and values) stay in L2, repeat reads are served "
                     "there and achieved can exceed the DRAM peak; traffic is the DRAM bytes "
                     "ncu measured (compulsory reads and the output); issue is the binding "
                     "resource, the kernel's warp instructions against the GPU's issue slots"),
        },
        "stages_ms": {"tree_build": t_tree / args.steps * 1e3,
                      "forward": t_fwd / args.steps * 1e3,
                      "tree_build_GBps": tree_bytes / (t_tree / args.steps) / 1e9},
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "how": "HostPipeline: every step copies Q, K, V, W in from pinned host memory "
                       "and its output back; the next step's copy-in and the previous step's "
                       "copy-out overlap this step's kernels on their own streams; L2 flushed "
                       "before every step's kernels inside the timed region"},
        "gpu_launches": args.steps * (tree_launches + 1),
        "clocks": clocks,
        "wall_s_timed_region": wall,
    }
    return line


def measured_hbm_peak() -> float:
    """hbm_gbs of MEASURED_PEAKS.json (the measured copy bandwidth), else the fallback 6650."""
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return 6650.0


def tree_build_launches(bh: int, n: int) -> int:
    """Kernel launches of one alhr_build_tree: the streaming launch takes levels 1..m1 from
    the keys (m1 = 5 below 2^24 keys in all, else 7; none below 16 keys), and every further
    launch up to 7 levels."""
    L = int(math.log2(n))
    if L < 4:
        return 1
    m1 = min(L, 5 if bh * n < (1 << 24) else 7)
    return 1 + math.ceil((L - m1) / 7)


def _event_time(fn, reps: int, flush) -> float:
    """Median seconds of fn() over reps, L2 flushed before each, CUDA events on the stream."""
    ts = []
    stream = torch.cuda.current_stream()
    for r in range(reps):
        flush.fill_(r & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(ts)


def run_stages(args):
    """Per-stage split of one step (tree build, predictor, route, unfused attend, and the fused
    forward that does the last three in one kernel), then the fused forward against N at fixed
    batch and heads (prefill of every position), with the fitted log-log exponent of its time."""
    from tree_routed_sparse_b200 import alhr, metrics, synth
    dev = torch.device("cuda", 0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 5)
    peak = measured_hbm_peak()
    alhr.set_launch_mode(args.launch_mode)

    def stages(wl):
        vb = max(-wl.qk_lo, wl.qk_hi)
        inp = synth.make_inputs(wl, dev)
        Q, K, V, W, bo = inp["Q"], inp["K"], inp["V"], inp["W"], inp["budget_override"]
        kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
                  score_bits=wl.score_bits, value_bound=vb)
        tree = alhr.build_tree(K, value_bound=vb)
        budget = bo if W is None else alhr.predict_budget(Q, K, tree, W, **kw)
        r = alhr.route(Q, K, tree, budget, with_expansions=False, **kw)
        idx, count = r["idx"], r["count"]
        out = torch.empty((wl.batch, wl.heads, wl.nq, wl.d), dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            alhr.forward(Q, K, V, tree, W=W, budget_override=bo, out=out, **kw)
        t = {"tree_build": _event_time(lambda: alhr.build_tree(K, tree, value_bound=vb), reps, flush)}
        if W is not None:
            t["predict_budget"] = _event_time(
                lambda: alhr.predict_budget(Q, K, tree, W, budget=budget, **kw), reps, flush)
        t["route"] = _event_time(lambda: alhr.route(Q, K, tree, budget, idx=idx, count=count,
                                                    with_expansions=False, **kw), reps, flush)
        akw = {k: v for k, v in kw.items() if k != "score_bits"}
        t["attend"] = _event_time(lambda: alhr.attend(Q, K, V, idx, count, out=out, **akw),
                                  reps, flush)
        t["fused_forward"] = _event_time(
            lambda: alhr.forward(Q, K, V, tree, W=W, budget_override=bo, out=out, **kw), reps, flush)
        full = alhr.forward(Q, K, V, tree, W=W, budget_override=bo, want_count=True,
                            want_expansions=True, want_budget=True, **kw)
        pos = np.broadcast_to(np.arange(wl.q_start, wl.q_start + wl.nq), (wl.bh, wl.nq))
        fb = metrics.forward_bytes(pos, wl.n, wl.d, wl.window, full["count"].cpu().numpy(),
                                   full["expansions"].cpu().numpy(), full["budget"].cpu().numpy(),
                                   wl.predictor, wl.max_keys, value_bound=vb)
        keys = float(count.float().mean())
        del inp, tree, out, idx, count, budget, full
        torch.cuda.empty_cache()
        return t, keys, fb

    base = synth.WORKLOADS[args.workload]
    t, keys, fb = stages(base)
    report = {"report": "stages", "workload": describe(base), "reps": reps,
              "launch_mode": args.launch_mode,
              "stage_ms": {k: v * 1e3 for k, v in t.items()}, "mean_keys_per_query": keys,
              "fused_forward_algorithmic_bytes": fb,
              "fused_forward_GBps": fb / t["fused_forward"] / 1e9, "peak_GBps": peak,
              "scaling": []}
    sweep = [] if args.no_sweep else [1024, 4096, 16384, 65536]
    for n in sweep:
        wl = base.replace(n=n, nq=n, q_start=0)
        t, keys, fb = stages(wl)
        q = wl.bh * wl.nq
        report["scaling"].append({"n": n, "queries": q, "fused_forward_ms": t["fused_forward"] * 1e3,
                                  "tree_build_ms": t["tree_build"] * 1e3,
                                  "ns_per_query": t["fused_forward"] / q * 1e9,
                                  "mean_keys_per_query": keys,
                                  "fused_forward_GBps": fb / t["fused_forward"] / 1e9,
                                  "frac_of_copy_peak": fb / t["fused_forward"] / 1e9 / peak})
    if sweep:
        xs = np.log([e["n"] for e in report["scaling"]])
        ys = np.log([e["fused_forward_ms"] for e in report["scaling"]])
        report["loglog_exponent_fused_forward_vs_n"] = float(np.polyfit(xs, ys, 1)[0])
    report["gpu"] = torch.cuda.get_device_name(dev)
    print(json.dumps(report))


def run_tree(args):
    """The tree build on the workload's keys: one JSON line with its time, its algorithmic bytes
    (keys read + tree block written) and their rate against the measured copy bandwidth."""
    from tree_routed_sparse_b200 import alhr, metrics, synth
    dev = torch.device("cuda", 0)
    wl = synth.WORKLOADS[args.workload]
    if args.batch:
        wl = wl.replace(batch=args.batch)
    vb = max(-wl.qk_lo, wl.qk_hi)
    K = synth.uniform_int8(wl.seed, synth.TID_K, (wl.batch, wl.heads, wl.n, wl.d), wl.qk_lo,
                           wl.qk_hi, dev)
    tree = torch.empty((wl.batch, wl.heads, alhr.tree_bytes(wl.n, wl.d, vb)), dtype=torch.uint8,
                       device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    run = lambda: alhr.build_tree(K, tree, value_bound=vb)
    for _ in range(args.warmup):
        run()
    t = _event_time(run, max(args.steps, 3), flush)
    nbytes = metrics.tree_bytes(wl.bh, wl.n, wl.d, vb)  # keys read + tree rows written
    peak = measured_hbm_peak()
    print(json.dumps({"report": "tree_build", "workload": describe(wl), "ms": t * 1e3,
                      "algorithmic_bytes": nbytes, "GBps": nbytes / t / 1e9,
                      "frac_of_copy_peak": nbytes / t / 1e9 / peak, "peak_GBps": peak,
                      "launches": tree_build_launches(wl.bh, wl.n),
                      "gpu": torch.cuda.get_device_name(dev)}))


def run_labels(args):
    """The phase-2 label kernel on the workload's Q and K: one JSON line with its time, the
    causal scores it ranks per second and the int8 tensor operations it issues."""
    from tree_routed_sparse_b200 import alhr, synth
    dev = torch.device("cuda", 0)
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl, dev)
    Q, K = inp["Q"], inp["K"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    shape = (wl.batch, wl.heads, wl.nq, 16)
    lab = torch.empty(shape, dtype=torch.int32, device=dev)
    sc = torch.empty(shape, dtype=torch.int32, device=dev)
    run = lambda: alhr.topk_labels(Q, K, k=16, q_start=wl.q_start, labels=lab, scores=sc)
    for _ in range(args.warmup):
        run()
    t = _event_time(run, max(args.steps, 3), flush)
    i = np.arange(wl.q_start, wl.q_start + wl.nq, dtype=np.float64)
    scores = float(wl.bh * (i + 1).sum())
    tiles = 0  # 128-query x 64-key tensor-core tiles issued (each up to the tile's last query)
    for q0 in range(0, wl.nq, 128):
        last = wl.q_start + min(q0 + 128, wl.nq) - 1
        tiles += last // 64 + 1
    mma_ops = 2.0 * wl.bh * tiles * 128 * 64 * wl.d
    print(json.dumps({"report": "labels", "workload": describe(wl), "k": 16,
                      "ms": t * 1e3, "queries_per_s": wl.bh * wl.nq / t,
                      "causal_scores_per_s": scores / t, "int8_tensor_tops": mma_ops / t / 1e12,
                      "gpu": torch.cuda.get_device_name(dev)}))


def profiled_record(workload: str):
    """The committed ncu record of the fused kernel on this workload (DRAM bytes and warp
    instructions per launch), if it was taken on the fused kernel's source (query_kernels.cu and
    the headers) as it is now; else None."""
    path = os.path.join(HERE, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    from tree_routed_sparse_b200 import build
    if rec.get("source_hash") != build.kernel_hash("query_kernels.cu"):
        return None
    return rec


# warp-instruction issue slots per second of one B200: 148 SMs x 4 schedulers x max SM clock
ISSUE_SLOTS_PER_S = 148 * 4 * 1965e6


def issue_rate(rec, launch_s: float):
    """The fused kernel's instruction issue against the GPU's issue slots: its warp
    instructions per launch (from the ncu record) over the live launch time, as a fraction of
    148 SMs x 4 schedulers x 1965 MHz. None without a current record."""
    if not rec or "warp_instructions_per_launch" not in rec:
        return None
    achieved = rec["warp_instructions_per_launch"] / launch_s
    return {"warp_instructions_per_launch": rec["warp_instructions_per_launch"],
            "achieved_per_s": achieved, "peak_per_s": ISSUE_SLOTS_PER_S,
            "frac": achieved / ISSUE_SLOTS_PER_S,
            "source": "instruction count from profiles/traffic.json (ncu), live launch time"}


def main():
    args = parse()
    if args.impl == "reference":
        # the oracle on the host cores; under torchrun only rank 0 works
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        from tree_routed_sparse_b200 import synth
        wl = synth.WORKLOADS[args.workload]
        inp = synth.make_inputs(wl, "cpu")
        all_blocks = [(b, h) for b in range(wl.batch) for h in range(wl.heads)]
        # one step = one (b,h) block (whole tree, every stride-th query row), round robin
        pick = lambda k: [all_blocks[j % len(all_blocks)] for j in range(k)]
        if args.warmup:
            oracle_sample(wl, args.ref_stride, pick(args.warmup), inp)
        r = oracle_sample(wl, args.ref_stride, pick(args.steps), inp)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wl.nq / r["value"] * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64",
            "data": "synthetic", "config": {"workload": describe(wl),
                                            "step": "one (b,h) block of the workload"},
            "cpu_baseline": {k: r[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": r["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }))
        return

    if args.labels:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        from tree_routed_sparse_b200 import build
        build.build()
        run_labels(args)
        return
    if args.tree:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        from tree_routed_sparse_b200 import build
        build.build()
        run_tree(args)
        return
    if args.stages:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        from tree_routed_sparse_b200 import build
        build.build()
        run_stages(args)
        return

    dist, rank, world = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    from tree_routed_sparse_b200 import build
    if rank == 0:
        build.build()
    barrier(dist)
    line = run_alhr(args, dist, rank, world)
    if rank == 0:
        if not args.no_cpu_baseline:
            from tree_routed_sparse_b200 import synth
            cb = oracle_sample(synth.WORKLOADS[args.workload], args.cpu_sample_stride)
            line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
