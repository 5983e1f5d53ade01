"""The (b, h)-sharded multi-GPU code path, run shard by shard on one GPU.

A weak-scaling run on `world` GPUs processes a global batch of world times the per-GPU
sequences; rank k draws its contiguous share of the (b, h) blocks from the seeded generator and
runs the tree build and the fused forward on them (bench.py's GPU arm does exactly this). Here
the shards of world = 2 and world = 3 run one after another on one GPU (no rank waits on
another, so nothing runs concurrently); their results, put side by side, must equal one
unsharded run over the whole global batch bit for bit, and sampled rows must match the oracle.
"""
import numpy as np
import pytest
import torch

from parity_util import compare_rows, oracle_slice

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def alhr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_routed_sparse_b200 import build
    build.build()
    from tree_routed_sparse_b200 import alhr as A
    A.lib()
    return A


def _run(alhr, wl, inp):
    vb = max(-wl.qk_lo, wl.qk_hi)
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits, value_bound=vb)
    tree = alhr.build_tree(inp["K"], value_bound=vb)
    res = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                       budget_override=inp["budget_override"], want_idx=True, want_count=True,
                       want_expansions=True, want_budget=True, **kw)
    torch.cuda.synchronize()
    return {k: v.reshape(-1, *v.shape[2:]).cpu() for k, v in res.items()}


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", ["prefill_b4h8_n4096", "recall_b2h4_n16384_d128"])
def test_shards_equal_the_unsharded_run(alhr, name, world):
    from tree_routed_sparse_b200 import shard, synth
    base = synth.WORKLOADS[name]
    per_gpu = base.replace(batch=1, heads=3, n=2048, nq=2048,
                           plant_pairs=min(base.plant_pairs, 64))
    g = shard.global_workload(per_gpu, world)
    dev = torch.device("cuda", 0)
    # the launch shape must not depend on the shard's size: force the throughput shape, as a
    # full-size launch takes
    alhr.set_launch_mode("throughput")
    try:
        _, _, whole_inp = shard.shard_inputs(g, 1, 0, dev)
        whole = _run(alhr, g, whole_inp)
        parts = []
        for r in range(world):
            lo, hi, inp = shard.shard_inputs(g, world, r, dev)
            assert lo == r * per_gpu.bh and hi == lo + per_gpu.bh
            parts.append(_run(alhr, g, inp))
    finally:
        alhr.set_launch_mode("auto")
    for key in whole:
        cat = torch.cat([p[key] for p in parts])
        assert torch.equal(cat, whole[key]), key
    # the oracle on sampled rows of the first block of every shard and the last block overall
    host = synth.make_inputs(g, "cpu")
    rows = np.unique(np.r_[np.arange(24), np.arange(100, 2048, 97), np.arange(2030, 2048)])
    blocks = [divmod(r * per_gpu.bh, g.heads) for r in range(world)] + [(g.batch - 1, g.heads - 1)]
    for b, h in blocks:
        ref = oracle_slice(host, g, b, h, rows=rows)
        flat = b * g.heads + h
        view = {k: v[flat:flat + 1].unsqueeze(0) for k, v in whole.items()}
        compare_rows(view, ref, 0, 0, rows, what=f"{name} world {world} block {(b, h)}")


def test_uneven_shards_split_a_sequence(alhr):
    """Blocks of one sequence on two ranks (6 blocks over 4 ranks): still the same results."""
    from tree_routed_sparse_b200 import shard, synth
    g = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=2, heads=3, n=1024, nq=1024)
    dev = torch.device("cuda", 0)
    alhr.set_launch_mode("throughput")
    try:
        whole = _run(alhr, g, shard.shard_inputs(g, 1, 0, dev)[2])
        parts = []
        for r in range(4):
            lo, hi, inp = shard.shard_inputs(g, 4, r, dev)
            assert inp["K"].shape[:2] == (1, hi - lo)
            parts.append(_run(alhr, g, inp))
    finally:
        alhr.set_launch_mode("auto")
    for key in whole:
        assert torch.equal(torch.cat([p[key] for p in parts]), whole[key]), key
