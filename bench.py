"""Benchmark of the ALHR inference path: routed queries per second on one step of the
configured workload (tree build + fused route/attend over every query), on N GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl alhr|reference]

N > 1 runs one process per GPU under torch.distributed.run (started by this script itself when
WORLD_SIZE is not set). Weak scaling: the global batch holds N times the workload's sequences
and rank k processes its contiguous share of the (b, h) blocks, drawn from the seeded generator
at their flat index in the global batch; no collective on the data path (NCCL carries only the
barrier and the max-over-ranks time). Prints one JSON line on rank 0. Inputs are seeded
synthetic tensors generated on the device; L2 is flushed by a 512 MiB write before every timed
step; the timed region holds exactly K steps bracketed by a barrier and a device
synchronisation; each step is timed with CUDA events on the launch stream and the job time is
the maximum over ranks.

--impl reference times the oracle (the plain CPU reference that the tests use) on the host
cores with the same metric: every step is one fully computed unit of the same workload (each
(b, h) block's tree and every R-th query row, rotating the offset from step to step), timed
as it runs; nothing is scaled.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import socket
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
L2_NOTE = "flushed by a 512 MiB write before every timed GPU step (not timed)"
# predictor classes kept live at the pages' operating point (rows of the higher classes are
# zero): the budget is then 3 (c + 1) with c uniform over 0..19, about 31 keys per query
OP_LIVE_CLASSES = 20


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="alhr", choices=["alhr", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--op-steps", type=int, default=100,
                    help="launches timed at the operating point of about 30 keys per query")
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
                    help="with --tree, --labels or --forward-only: replace the workload's batch "
                         "(sequences)")
    ap.add_argument("--n", type=int, default=0,
                    help="with --forward-only: replace the workload's sequence length (decode "
                         "workloads keep their one query at position n-1)")
    ap.add_argument("--forward-only", action="store_true",
                    help="instead of the bench line: time the fused forward (tree prebuilt, L2 "
                         "flushed before each launch) on the workload, e.g. one decode launch")
    ap.add_argument("--cpu-steps", type=int, default=4,
                    help="CPU baseline: oracle steps on all host cores (each as a reference step)")
    ap.add_argument("--row-stride", type=int, default=16,
                    help="oracle steps: every R-th query row of every (b,h) block, the first "
                         "row rotating with the step")
    ap.add_argument("--no-single-thread", action="store_true",
                    help="CPU baseline: skip the single-threaded full-block timing")
    return ap.parse_args(argv)


def describe(wl) -> str:
    pred = (f"predictor W int8 U[{wl.w_lo},{wl.w_hi}] 32x{2 * wl.d}" if wl.predictor
            else f"fixed budget min(i+1,{wl.fixed_budget_cap})")
    if wl.predictor and wl.live_classes < 32:
        pred += f" with classes >= {wl.live_classes} zeroed"
    extra = f", {wl.plant_pairs} planted pairs/seq" if wl.plant_pairs else ""
    return (f"{wl.name}: batch {wl.batch}, heads {wl.heads}, N={wl.n}, d={wl.d}, "
            f"queries [{wl.q_start},{wl.q_start + wl.nq}), w={wl.window}, max_keys={wl.max_keys}, "
            f"Q/K int8 U[{wl.qk_lo},{wl.qk_hi}], V bf16 N(0,1), {pred}{extra}")


def bench_config(wl) -> dict:
    """The `config` object, identical in both arms: the per-GPU workload and the L2 policy."""
    return {"workload": describe(wl), "l2": L2_NOTE}


# ------------------------------------------------------------------ distributed plumbing

def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun_command(argv: list[str], n: int, port: int) -> list[str]:
    """The command that runs this script with the same arguments as n ranks, one per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def dist_setup(n_gpus: int):
    """(dist module or None, rank, world) for a run under torch.distributed.run; the world size
    must equal --gpus."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE {world}")
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
    """SM clocks and clock-event (throttle) reasons sampled during the timed region: through NVML
    from a thread every 2 ms (the timed region can be well under a second), else through
    nvidia-smi every 200 ms. Read-only: no setting of the GPU is touched."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.thread = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, reasons set)
        self.how = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._nvml_index())
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.stop_flag = False

            def poll():
                while not self.stop_flag:
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, mx, {k for k, b in bits.items() if r & b}))
                    except Exception:  # noqa: BLE001 - sampling must never stop the bench
                        pass
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.how = "NVML, every 2 ms"
            return
        except Exception:  # noqa: BLE001 - no NVML: fall back to nvidia-smi
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            self.how = "nvidia-smi, every 200 ms"
        except OSError:
            self.proc = None

    def _nvml_index(self) -> int:
        """NVML index of the CUDA device (CUDA_VISIBLE_DEVICES may renumber them)."""
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [v.strip() for v in vis.split(",") if v.strip()]
            if self.dev < len(ids) and ids[self.dev].isdigit():
                return int(ids[self.dev])
        return self.dev

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=2)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=2)
            for ln in self.lines:
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm, mx = float(f[1]), float(f[2])
                except ValueError:
                    continue
                self.samples.append((sm, mx, {nm for nm, v in zip(self.NAMES, f[5:9])
                                              if v.lower() == "active"}))
        if not self.samples:
            return None
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(x[0] for x in self.samples),
                "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(self.samples), "how": self.how}


# ------------------------------------------------------------------ oracle (CPU) timing

def _host_blocks(inp):
    """Per-(b,h) numpy views of host inputs."""
    Vbits = inp["V"].view(torch.int16).numpy().view(np.uint16)
    W = None if inp["W"] is None else inp["W"].numpy()
    return Vbits, W


def oracle_steps(wl, inp, steps: int, row_stride: int, first_step: int = 0) -> dict:
    """The oracle as it stands on the host cores, step by step. Step s is one fully computed
    unit of the workload: for every (b,h) block, its tree and the query rows r with
    r = (first_step + s) mod R (mod R), R = min(row_stride, nq), so R consecutive steps cover
    every row once. Blocks run on a thread pool, one block per thread (the oracle is
    single-threaded; ctypes releases the GIL). Each step's wall time is measured as it runs;
    the value is the queries computed over the summed step times."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as orc

    orc.lib()
    blocks = [(b, h) for b in range(wl.batch) for h in range(wl.heads)]
    R = max(1, min(row_stride, wl.nq))
    Vbits, W = _host_blocks(inp)

    def run(arg):
        (b, h), rows = arg
        bo = None if inp["budget_override"] is None else inp["budget_override"][b, h].numpy()
        nodes = orc.build_tree(inp["K"][b, h].numpy())
        orc.forward(inp["Q"][b, h].numpy(), inp["K"][b, h].numpy(), Vbits[b, h], nodes, W, bo,
                    q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys, rows=rows)

    threads = max(1, min(os.cpu_count() or 1, len(blocks)))
    times, queries = [], 0
    with ThreadPoolExecutor(threads) as ex:
        for s in range(steps):
            rows = np.arange((first_step + s) % R, wl.nq, R, dtype=np.int32)
            t0 = time.perf_counter()
            list(ex.map(run, [(bh, rows) for bh in blocks]))
            times.append(time.perf_counter() - t0)
            queries += len(rows) * len(blocks)
    total = sum(times)
    return {"value": queries / total if total > 0 else 0.0, "unit": "queries/s",
            "cores": threads, "kind": "oracle", "step_s": times, "queries": queries,
            "sample": (f"{describe(wl)}; {steps} step(s), each: the tree of every one of the "
                       f"{len(blocks)} (b,h) blocks plus every {R}-th query row of it (rows "
                       f"r = step mod {R}), {queries} queries in all, fully computed and timed "
                       f"as run (no scaling); {threads} threads, one block per thread")}


def oracle_single_thread(wl, inp) -> dict:
    """The single-threaded oracle figure: block (b,h) = (0,0), its tree and every query row,
    timed with std::chrono::steady_clock inside the oracle library on one thread."""
    from oracle import oracle as orc
    Vbits, W = _host_blocks(inp)
    bo = None if inp["budget_override"] is None else inp["budget_override"][0, 0].numpy()
    t, _ = orc.time_block(inp["Q"][0, 0].numpy(), inp["K"][0, 0].numpy(), Vbits[0, 0], W, bo,
                          wl.q_start, wl.window, wl.max_keys)
    return {"value": wl.nq / t, "unit": "queries/s", "cores": 1, "kind": "oracle",
            "block_s": t, "us_per_query": t / wl.nq * 1e6,
            "sample": (f"(b,h) = (0,0) of {wl.name}: its tree and all {wl.nq} queries, one "
                       "thread, std::chrono::steady_clock inside the oracle library")}


# ------------------------------------------------------------------ the GPU arm

# The latency shape (one query per CTA) takes launches whose queries are all resident at once:
# four warps per query up to 4 CTAs per SM, two warps per query up to 8 per SM (7 where shared
# memory runs out first); larger launches take the warp-per-query shape.
LAT_CTAS_PER_SM = 8


def takes_warp_shape(queries: int, dev) -> bool:
    return queries > torch.cuda.get_device_properties(dev).multi_processor_count * LAT_CTAS_PER_SM


def fwd_algorithmic_bytes(wl, full, vb, warp_shape: bool = True) -> tuple[int, int]:
    """(algorithmic bytes, bytes of the rows the kernel reads) of one fused-forward launch. The
    first is the byte model as the method defines it (G_i from the forest roots and the window
    keys); the second differs only where the warp-per-query kernel at d = 64 forms G_i from the
    blocks of [0, i+1) instead."""
    from tree_routed_sparse_b200 import metrics
    pos = np.broadcast_to(np.arange(wl.q_start, wl.q_start + wl.nq),
                          (full["count"].shape[0] * full["count"].shape[1], wl.nq))
    args = (pos, wl.n, wl.d, wl.window, full["count"].cpu().numpy(),
            full["expansions"].cpu().numpy(), full["budget"].cpu().numpy(), wl.predictor,
            wl.max_keys)
    plain = metrics.forward_bytes(*args, value_bound=vb)
    kernel = metrics.forward_bytes(*args, value_bound=vb,
                                   g_from_blocks=warp_shape and wl.d == 64)
    return plain, kernel


def run_alhr(args, dist, rank, world):
    from tree_routed_sparse_b200 import alhr, metrics, shard, synth
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.WORKLOADS[args.workload]
    wlg = shard.global_workload(wl, world)
    lo, hi, inp = shard.shard_inputs(wlg, world, rank, dev)
    assert hi - lo == wl.bh and inp["K"].shape[:2] == (wl.batch, wl.heads)
    vb = max(-wl.qk_lo, wl.qk_hi)
    Q, K, V, W, bo = inp["Q"], inp["K"], inp["V"], inp["W"], inp["budget_override"]
    tree = torch.empty((wl.batch, wl.heads, alhr.tree_bytes(wl.n, wl.d, vb)), dtype=torch.uint8,
                       device=dev)
    out = torch.empty((wl.batch, wl.heads, wl.nq, wl.d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits, value_bound=vb)
    path_bytes = sum(t.numel() * t.element_size() for t in (Q, K, V, W, bo, tree, out)
                     if t is not None)
    sbits = 32 if alhr.score_bits(alhr.make_dims(Q, K, **kw)) == 32 else 64

    # one untimed run with every output: counts for the byte model
    alhr.build_tree(K, tree, value_bound=vb)
    full = alhr.forward(Q, K, V, tree, W=W, budget_override=bo, want_count=True,
                        want_expansions=True, want_budget=True, **kw)
    torch.cuda.synchronize()
    warp_shape = takes_warp_shape(wl.bh * wl.nq, dev)
    fwd_bytes, fwd_kernel_bytes = fwd_algorithmic_bytes(wl, full, vb, warp_shape)
    tree_bytes = metrics.tree_bytes(wl.bh, wl.n, wl.d, vb)
    mean_keys = float(full["count"].float().mean())
    mean_budget = float(full["budget"].float().mean())
    del full

    for _ in range(args.warmup):
        flush.fill_(1)
        alhr.build_tree(K, tree, value_bound=vb)
        alhr.forward(Q, K, V, tree, W=W, budget_override=bo, out=out, **kw)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    torch.cuda.reset_peak_memory_stats(dev)
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
    peak_alloc = torch.cuda.max_memory_allocated(dev)
    t_tree = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_fwd = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    out_ref = out.cpu()  # the step's output, which the end-to-end run must reproduce
    t_step = t_tree + t_fwd
    t_job = max_over_ranks(dist, t_step)
    queries = wl.bh * wl.nq
    value = world * queries * args.steps / t_job

    # the pages' operating point (about 30 keys read per query): the same inputs, predictor
    # rows of classes >= OP_LIVE_CLASSES zeroed; fused forward only (the tree is unchanged)
    op = None
    if W is not None and args.op_steps > 0:
        W_op = W.clone()
        W_op[OP_LIVE_CLASSES:] = 0
        wl_op = wl.replace(live_classes=OP_LIVE_CLASSES)
        full = alhr.forward(Q, K, V, tree, W=W_op, want_count=True, want_expansions=True,
                            want_budget=True, **kw)
        torch.cuda.synchronize()
        op_bytes, op_kernel_bytes = fwd_algorithmic_bytes(wl_op, full, vb, warp_shape)
        op_keys = float(full["count"].float().mean())
        del full
        for _ in range(3):
            alhr.forward(Q, K, V, tree, W=W_op, out=out, **kw)
        evo = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
               for _ in range(args.op_steps)]
        barrier(dist)
        torch.cuda.synchronize()
        for s in range(args.op_steps):
            flush.fill_(s & 0xFF)
            evo[s][0].record(stream)
            alhr.forward(Q, K, V, tree, W=W_op, out=out, **kw)
            evo[s][1].record(stream)
        torch.cuda.synchronize()
        t_op = max_over_ranks(dist, sum(e[0].elapsed_time(e[1]) for e in evo) / 1e3)
        op = {"workload": describe(wl_op), "mean_keys_per_query": op_keys,
              "pages_keys_per_token": "30.0 / 32.0 / 30.0 at T = 1K / 4K / 16K (README TLDR)",
              "queries_per_s": world * queries * args.op_steps / t_op,
              "launch_ms": t_op / args.op_steps * 1e3, "algorithmic_bytes_per_launch": op_bytes,
              "kernel_row_bytes_per_launch": op_kernel_bytes}

    # end to end through the public API, host buffers: every step copies its inputs in from
    # pinned memory, builds the tree, runs the fused forward and copies the output back, through
    # tree_routed_sparse_b200.pipeline.HostPipeline (copies of the next and the previous step
    # overlap this step's kernels on their own streams; L2 flushed on the compute stream before
    # every step, inside the timed region). The device tensors of the runs above are freed
    # first; a workload whose double-buffered pipeline does not fit runs single-buffered, and the
    # number of steps is capped at about two seconds of copies.
    from tree_routed_sparse_b200.pipeline import HostPipeline
    import psutil
    h2d = sum(v.numel() * v.element_size() for v in inp.values() if v is not None)
    d2h = out_ref.numel() * out_ref.element_size()
    e2e_skip = None
    if h2d > (8 << 30):
        e2e_skip = (f"a step's inputs are {h2d / 2**30:.0f} GiB: the end-to-end run (all inputs "
                    "copied in from pinned host memory every step) is measured for workloads of "
                    "at most 8 GiB per step")
    elif 3 * h2d > psutil.virtual_memory().available:
        e2e_skip = "not enough free host memory to pin a copy of the inputs"
    if e2e_skip is None:
        host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in inp.items()}
    del inp, Q, K, V, W, bo, tree, out
    torch.cuda.empty_cache()
    nbuf, e2e_steps, e2e_value = 0, 0, None
    if e2e_skip is None:
        outs_host = [torch.empty(out_ref.shape, dtype=out_ref.dtype).pin_memory()
                     for _ in range(2)]
        free, _ = torch.cuda.mem_get_info(dev)
        nbuf = 2 if 2 * path_bytes < 0.9 * free else 1
        e2e_steps = max(3, min(args.e2e_steps, int(2.0 / max((h2d + d2h) / 50e9, 1e-6))))
        pipe = HostPipeline(host, device=dev, flush=flush, buffers=nbuf, **kw)
        for s in range(3):
            pipe.submit(host, outs_host[s & 1])
        pipe.synchronize()
        assert torch.equal(outs_host[0], out_ref) and torch.equal(outs_host[1], out_ref)
    # every rank takes the same collective steps, measured or not
    barrier(dist)
    torch.cuda.synchronize()
    t_e2e = 0.0
    if e2e_skip is None:
        e2e_start = torch.cuda.Event(enable_timing=True)
        e2e_end = torch.cuda.Event(enable_timing=True)
        e2e_start.record(pipe.copy_in)
        for s in range(e2e_steps):
            pipe.submit(host, outs_host[s & 1])
        e2e_end.record(pipe.copy_out)
        pipe.synchronize()
        t_e2e = e2e_start.elapsed_time(e2e_end) / 1e3
        del pipe, host, outs_host
    barrier(dist)
    t_e2e = max_over_ranks(dist, t_e2e)
    if e2e_skip is None:
        e2e_value = world * queries * e2e_steps / t_e2e

    if rank != 0:
        return None

    peak = measured_hbm_peak()
    peak_src = "measured" if peak_is_measured() else "fallback"
    fwd_launch_s = t_fwd / args.steps
    achieved = fwd_bytes / fwd_launch_s / 1e9
    rec = profiled_record(args.workload)
    traffic = rec.get("dram_bytes_per_launch") if rec else None
    tree_launches = tree_build_launches(wl.bh, wl.n)
    if op is not None:
        op_rec = profiled_record(f"{args.workload}+live{OP_LIVE_CLASSES}")
        op_s = op["launch_ms"] / 1e3
        op["algorithmic_GBps"] = op["algorithmic_bytes_per_launch"] / op_s / 1e9
        op["frac_of_measured_hbm"] = op["algorithmic_GBps"] / peak
        op["issue"] = issue_rate(op_rec, op_s)
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
        "config": bench_config(wl),
        "step": "alhr_build_tree + alhr_forward (fused budget, window, descent, attention)",
        "parallelism": (f"{world} GPU(s): a global batch of {wlg.batch} sequences x {wl.heads} "
                        f"heads, each rank its contiguous {wl.bh} (b,h) blocks; no collective "
                        "on the data path"),
        "queries_per_step_per_gpu": queries,
        "score_bits": sbits,
        "mean_keys_per_query": mean_keys,
        "mean_budget": mean_budget,
        "roofline": {
            "bound": "hbm",
            "kernel": "query_kernel (fused alhr_forward)",
            "achieved": achieved,
            "peak": peak,
            "unit": "GB/s",
            "frac": achieved / peak,
            "peak_source": f"{peak_src} hbm_gbs",
            "algorithmic_bytes_per_launch": fwd_bytes,
            "kernel_row_bytes_per_launch": fwd_kernel_bytes,
            "launch_ms": fwd_launch_s * 1e3,
            "traffic": traffic,
            "dram": dram_rate(traffic, fwd_launch_s, peak),
            "issue": issue_rate(rec, fwd_launch_s),
            "binding_resource": "instruction issue (see issue.frac); DRAM is not the limit",
            "note": ("achieved counts every row the method reads (the algorithmic bytes: G_i from "
                     "the forest roots and the window keys) as if it came from DRAM; "
                     "kernel_row_bytes are the rows the kernel reads (at d = 64 it forms G_i from "
                     "the blocks of [0, i+1), a few more rows); queries run in (b, h, i) order, so the "
                     "rows in use at any time (about one head's tree, keys and values) stay in "
                     "L2 and repeat reads are served there: achieved is a rate of row reads and "
                     "can exceed the DRAM peak. dram is the DRAM traffic ncu measured "
                     "(compulsory reads and the output) over the same launch time; issue is "
                     "the binding resource, the kernel's warp instructions against the GPU's "
                     "issue slots"),
        },
        "stages_ms": {"tree_build": t_tree / args.steps * 1e3,
                      "forward": t_fwd / args.steps * 1e3,
                      "tree_build_GBps": tree_bytes / (t_tree / args.steps) / 1e9},
        "memory": {"peak_allocated_bytes": peak_alloc,
                   "path_bytes": path_bytes,
                   "l2_flush_buffer_bytes": L2_FLUSH_BYTES,
                   "note": ("peak_allocated_bytes: torch.cuda.max_memory_allocated over the "
                            "timed steps (the step's inputs, tree and output, plus the L2 flush "
                            "buffer); the library itself allocates nothing")},
        "operating_point_30_keys": op,
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "skipped": e2e_skip,
                "how": None if e2e_skip else (
                    "HostPipeline: every step copies Q, K, V, W in from pinned host memory and "
                    "its output back; " + (
                        "the next step's copy-in and the previous step's copy-out overlap this "
                        "step's kernels on their own streams" if nbuf == 2 else
                        "single-buffered (two device copies of the step do not fit): the copies "
                        "wait for the kernels") +
                    "; L2 flushed before every step's kernels inside the timed region")},
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


def peak_is_measured() -> bool:
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            return "hbm_gbs" in json.load(f)
    except (OSError, ValueError):
        return False


def dram_rate(traffic, launch_s: float, peak: float):
    """DRAM bytes per launch (ncu) over the live launch time, against the measured copy peak."""
    if not traffic:
        return None
    gbps = traffic / launch_s / 1e9
    return {"bytes_per_launch": traffic, "GBps": gbps, "frac": gbps / peak,
            "source": "dram__bytes_read.sum + dram__bytes_write.sum from profiles/traffic.json "
                      "(ncu), live launch time"}


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
        fb, _ = fwd_algorithmic_bytes(wl, full, vb)
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


def override_workload(wl, args):
    """The workload with --batch / --n applied (a decode workload keeps its query at n-1)."""
    if args.batch:
        wl = wl.replace(batch=args.batch)
    if args.n:
        if wl.nq == 1 and wl.q_start == wl.n - 1:
            wl = wl.replace(n=args.n, q_start=args.n - 1)
        else:
            wl = wl.replace(n=args.n, nq=args.n, q_start=0)
    return wl


def run_forward_only(args):
    """The fused forward alone (tree prebuilt), L2 flushed before every launch: one JSON line with
    the median launch time, queries per second and the algorithmic bytes' rate."""
    from tree_routed_sparse_b200 import alhr, synth
    dev = torch.device("cuda", 0)
    alhr.set_launch_mode(args.launch_mode)
    wl = override_workload(synth.WORKLOADS[args.workload], args)
    vb = max(-wl.qk_lo, wl.qk_hi)
    inp = synth.make_inputs(wl, dev)
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits, value_bound=vb)
    tree = alhr.build_tree(inp["K"], value_bound=vb)
    out = torch.empty((wl.batch, wl.heads, wl.nq, wl.d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    run = lambda: alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                               budget_override=inp["budget_override"], out=out, **kw)
    for _ in range(args.warmup):
        run()
    t = _event_time(run, max(args.steps, 3), flush)
    full = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                        budget_override=inp["budget_override"], want_count=True,
                        want_expansions=True, want_budget=True, **kw)
    torch.cuda.synchronize()
    fb, kb = fwd_algorithmic_bytes(wl, full, vb, takes_warp_shape(wl.bh * wl.nq, dev)
                                   if args.launch_mode == "auto" else args.launch_mode == "throughput")
    q = wl.bh * wl.nq
    print(json.dumps({"report": "forward", "workload": describe(wl), "launch_mode": args.launch_mode,
                      "queries": q, "us": t * 1e6, "queries_per_s": q / t,
                      "mean_keys_per_query": float(full["count"].float().mean()),
                      "algorithmic_bytes": fb, "kernel_row_bytes": kb,
                      "algorithmic_GBps": fb / t / 1e9, "gpu": torch.cuda.get_device_name(dev)}))


def run_labels(args):
    """The phase-2 label kernel on the workload's Q and K: one JSON line with its time, the
    causal scores it ranks per second and the int8 tensor operations it issues."""
    from tree_routed_sparse_b200 import alhr, synth
    dev = torch.device("cuda", 0)
    wl = override_workload(synth.WORKLOADS[args.workload], args)
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


def run_reference(args):
    """The reference arm: the oracle on the host cores, rank 0 only, K timed steps after W
    warm-up steps, each step a fully computed unit of the same workload (oracle_steps)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl, "cpu")
    if args.warmup:
        oracle_steps(wl, inp, args.warmup, args.row_stride)
    r = oracle_steps(wl, inp, args.steps, args.row_stride, first_step=args.warmup)
    cb = {k: r[k] for k in ("value", "unit", "cores", "kind", "sample")}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(r["step_s"]) / max(1, len(r["step_s"])) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64",
        "data": "synthetic (seeded SplitMix64; random int8 predictor weights, no trained model)",
        "config": bench_config(wl),
        "step": ("the oracle (tree build + whole path) on every (b,h) block's tree and every "
                 f"{max(1, min(args.row_stride, wl.nq))}-th query row, fully computed"),
        "queries_per_step": r["queries"] // max(1, args.steps),
        "cpu_baseline": cb,
        "e2e": {"value": r["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def cpu_baseline(args) -> dict:
    """The GPU arm's CPU baseline (rank 0, N = 1 line): the reference arm's procedure for
    --cpu-steps steps on all host cores, plus the single-threaded full-block figure."""
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl, "cpu")
    r = oracle_steps(wl, inp, args.cpu_steps, args.row_stride)
    cb = {k: r[k] for k in ("value", "unit", "cores", "kind", "sample")}
    if not args.no_single_thread:
        cb["single_thread"] = oracle_single_thread(wl, inp)
    return cb


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        run_reference(args)
        return
    if args.labels or args.tree or args.stages or args.forward_only:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device")
        from tree_routed_sparse_b200 import build
        build.build()
        (run_labels if args.labels else run_tree if args.tree else
         run_forward_only if args.forward_only else run_stages)(args)
        return

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start this script again under torch.distributed.run
        if not torch.cuda.is_available() or torch.cuda.device_count() < args.gpus:
            raise SystemExit(f"--gpus {args.gpus}: only "
                             f"{torch.cuda.device_count() if torch.cuda.is_available() else 0} "
                             "CUDA device(s) visible")
        from tree_routed_sparse_b200 import build
        build.build()  # once, before the ranks start
        argv = sys.argv[1:] if argv is None else list(argv)
        rc = subprocess.run(torchrun_command(argv, args.gpus, free_port())).returncode
        raise SystemExit(rc)

    dist, rank, world = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    from tree_routed_sparse_b200 import build
    if rank == 0:
        build.build()
    barrier(dist)
    line = run_alhr(args, dist, rank, world)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args)
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
