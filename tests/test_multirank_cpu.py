"""Two host ranks over gloo: each processes its shard of the (b, h) blocks of one batch with the
oracle; the gathered result must equal a single-process run, and the job time is the maximum
over ranks. No GPU is involved."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

from tree_routed_sparse_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path[:0] = [ROOT, os.path.join(ROOT, "tests")]
    import datetime
    import torch.distributed as dist
    import bench
    from parity_util import oracle_slice
    from tree_routed_sparse_b200 import shard as sh, synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=2, heads=3, n=128, nq=128)
    inp = synth.make_inputs(wl, "cpu")
    mine = {}
    for b, h in sh.blocks_of(wl.batch, wl.heads, world, rank):
        r = oracle_slice(inp, wl, b, h)
        mine[(b, h)] = (r["idx"], r["count"], r["out"])
    gathered = [None] * world
    dist.all_gather_object(gathered, mine)
    t = bench.max_over_ranks(dist, 0.5 + rank)
    if rank == 0:
        merged = {}
        for part in gathered:
            merged.update(part)
        q.put((merged, t))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("total,world", [(6, 2), (7, 3), (16, 1), (3, 4), (0, 2)])
def test_shard_ranges_cover_once(total, world):
    seen = []
    for r in range(world):
        lo, hi = shard.shard_range(total, world, r)
        assert 0 <= hi - lo <= total // world + 1
        seen += list(range(lo, hi))
    assert seen == list(range(total))


def test_two_gloo_ranks_match_single_process():
    import sys
    sys.path[:0] = [os.path.join(ROOT, "tests")]
    from parity_util import oracle_slice
    from tree_routed_sparse_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged, t = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert t == 1.5
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=2, heads=3, n=128, nq=128)
    inp = synth.make_inputs(wl, "cpu")
    assert sorted(merged) == [(b, h) for b in range(2) for h in range(3)]
    for (b, h), (idx, count, out) in merged.items():
        r = oracle_slice(inp, wl, b, h)
        assert np.array_equal(idx, r["idx"]) and np.array_equal(count, r["count"])
        assert np.array_equal(out, r["out"])


def _bench_shard_worker(rank, world, port, q):
    """As bench.py's GPU arm shards its global batch, on the host: rank k draws its blocks with
    shard.shard_inputs, runs the oracle on them, and the gathered blocks must be the global
    batch's blocks in order."""
    import sys
    sys.path[:0] = [ROOT, os.path.join(ROOT, "tests")]
    import datetime
    import torch.distributed as dist
    import bench
    from parity_util import oracle_slice
    from tree_routed_sparse_b200 import shard as sh, synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    per_gpu = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=3, n=128, nq=128)
    g = sh.global_workload(per_gpu, world)
    lo, hi, inp = sh.shard_inputs(g, world, rank)
    mine = {}
    for b in range(inp["K"].shape[0]):
        for h in range(inp["K"].shape[1]):
            flat = lo + b * inp["K"].shape[1] + h
            r = oracle_slice(inp, g, b, h)
            mine[flat] = (inp["K"][b, h].numpy().copy(), r["idx"], r["out"])
    gathered = [None] * world
    dist.all_gather_object(gathered, mine)
    t = bench.max_over_ranks(dist, 1.0 + 0.25 * rank)
    if rank == 0:
        merged = {}
        for part in gathered:
            merged.update(part)
        q.put((merged, t))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_a_global_batch():
    import sys
    sys.path[:0] = [os.path.join(ROOT, "tests")]
    from parity_util import oracle_slice
    from tree_routed_sparse_b200 import shard as sh, synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged, t = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert t == 1.25
    per_gpu = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=3, n=128, nq=128)
    g = sh.global_workload(per_gpu, 2)
    full = synth.make_inputs(g, "cpu")
    assert sorted(merged) == list(range(g.bh))
    for flat, (K, idx, out) in merged.items():
        b, h = divmod(flat, g.heads)
        assert np.array_equal(K, full["K"][b, h].numpy())
        ref = oracle_slice(full, g, b, h)
        assert np.array_equal(idx, ref["idx"]) and np.array_equal(out, ref["out"])
