"""Parity at the benchmark table's full sizes, in the benchmark's launch configuration.

Each workload runs once exactly as the benchmark times it (tree build, then the fused forward
with only `out` requested) and once with every optional output; `out` must be identical between
the two. Sampled (b, h) blocks are then checked against the oracle on sampled query rows that
include the first positions, the last positions (the ragged end of the grid) and a stride in
between: tree sums, budgets, index sets, counts and expansions bit-exact, outputs within 1e-3.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_util import compare_rows, decode_tree, oracle_slice

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def alhr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_routed_sparse_b200 import build
    build.build()
    from tree_routed_sparse_b200 import alhr as A
    A.lib()
    return A


def _sample_rows(nq, rng, k=40):
    if nq <= 3 * k:
        return np.arange(nq)
    mid = rng.choice(np.arange(k, nq - k), size=k, replace=False)
    return np.unique(np.r_[np.arange(k // 2), mid, np.arange(nq - k // 2, nq)])


def _slice_inputs(inp, wl, b, h):
    """Host copies of one (b, h) block (plus W / budget), as oracle_slice expects."""
    cut = lambda t: None if t is None else t[b:b + 1, h:h + 1].cpu()
    return dict(Q=cut(inp["Q"]), K=cut(inp["K"]), V=cut(inp["V"]),
                W=None if inp["W"] is None else inp["W"].cpu(),
                budget_override=cut(inp["budget_override"]))


@pytest.mark.parametrize("name,blocks", [
    ("tiny_prefill_n1024", [(0, 0)]),
    ("prefill_b4h8_n4096", [(0, 0), (3, 7)]),
    ("prefill_b2h8_n16384", [(0, 3), (1, 7)]),
    ("prefill_b2h8_n65536", [(0, 5), (1, 2)]),
    ("recall_b2h4_n16384_d128", [(0, 0), (1, 3)]),
    ("decode_s64h8_n262144_d128", [(0, 0), (5, 1), (17, 2), (31, 3), (40, 4), (50, 5),
                                   (62, 6), (63, 7)]),
])
def test_workload_parity(alhr, name, blocks):
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS[name]
    need = wl.bh * wl.n * wl.d * (1 + 2 + 4) + wl.bh * wl.nq * wl.d * 5  # K, V, tree <= 4d/row
    free, _ = torch.cuda.mem_get_info()
    if need > free - (2 << 30):
        pytest.skip(f"{name} needs {need / 2**30:.1f} GiB, {free / 2**30:.1f} GiB free")
    inp = synth.make_inputs(wl, "cuda")
    vb = max(-wl.qk_lo, wl.qk_hi)
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits, value_bound=vb)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the benchmark's configuration
    tree = alhr.build_tree(inp["K"], value_bound=vb, dev_err=err)
    bench_out = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                             budget_override=inp["budget_override"], dev_err=err, **kw)["out"]
    full = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                        budget_override=inp["budget_override"], want_idx=True, want_count=True,
                        want_expansions=True, want_budget=True, dev_err=err, **kw)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(bench_out, full["out"])
    rng = np.random.default_rng(0)
    for b, h in blocks:
        rows = _sample_rows(wl.nq, rng)
        cpu = _slice_inputs(inp, wl, b, h)
        ref = oracle_slice(cpu, wl, 0, 0, rows=rows)
        got = decode_tree(tree[b, h].cpu().numpy(), wl.n, wl.d, vb)
        assert np.array_equal(got, ref["nodes"]), f"tree {b},{h}"
        sub = {k: v[b:b + 1, h:h + 1].cpu() for k, v in full.items()}
        compare_rows(sub, ref, 0, 0, rows, TOL, f"{name} b{b}h{h}")
    if wl.plant_pairs:
        # diagnostic only: how often the planted key lands in its query's selection
        hits = 0
        idx = full["idx"].cpu()
        for b in range(wl.batch):
            p, u = synth.plant_positions(wl, b)
            sel = idx[b][:, u]  # [H, P, max_keys]
            hits += int((sel == p.view(1, -1, 1).to(torch.int32)).any(-1).sum())
        print(f"recall@selection {hits / (wl.batch * wl.heads * wl.plant_pairs):.3f}")
    del inp, tree, full, bench_out
    torch.cuda.empty_cache()


def test_largest_sequence_decode_and_update(alhr):
    """n = 2^20 keys (the largest the layout supports, 20 tree levels), d = 128, int64 scores:
    the tree against the oracle, decode-style queries at the end of the sequence against the
    oracle in both launch shapes, and a one-key update against a full build."""
    from tree_routed_sparse_b200 import synth
    n = 1 << 20
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(batch=1, heads=2, n=n,
                                                              q_start=n - 4, nq=4, seed=20)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"])
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys,
              score_bits=wl.score_bits)
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    tc = tree.cpu().numpy()
    for h in range(wl.heads):
        nodes = orc.build_tree(cpu["K"][0, h].numpy())
        assert np.array_equal(decode_tree(tc[0, h], n, wl.d), nodes), h
        ref = oracle_slice(cpu, wl, 0, h, nodes=nodes)
        for shape in ("latency", "throughput"):
            alhr.set_launch_mode(shape)
            try:
                res = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"], want_idx=True,
                                   want_count=True, want_expansions=True, want_budget=True,
                                   **kw)
                torch.cuda.synchronize()
            finally:
                alhr.set_launch_mode("auto")
            compare_rows(res, ref, 0, h, np.arange(wl.nq), TOL, f"n=2^20 {shape} h{h}")
    K2 = inp["K"].clone()
    K2[:, :, n - 1] = -K2[:, :, n - 1]
    alhr.update_tree(K2, tree, n - 1, n)
    assert torch.equal(tree, alhr.build_tree(K2))


@pytest.mark.parametrize("d,bits", [(128, 64), (64, 32)])
def test_mid_size_decode_launch(alhr, d, bits):
    """768 decode queries: more than the four-warp CTA shape holds at once on a B200 (4 per SM),
    so the latency shape runs two warps per query; auto and forced latency mode both take it.
    Sampled blocks against the oracle (bit-exact index sets, budgets, counts, expansions)."""
    from tree_routed_sparse_b200 import synth
    n = 4096
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(batch=96, n=n, d=d, q_start=n - 1,
                                                              score_bits=bits, seed=5)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"])
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys, score_bits=bits)
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    rng = np.random.default_rng(3)
    blocks = [(0, 0), (95, 7)] + [tuple(x) for x in zip(rng.integers(0, 96, 10),
                                                        rng.integers(0, 8, 10))]
    refs = {bh: oracle_slice(cpu, wl, bh[0], bh[1]) for bh in blocks}
    for shape in ("auto", "latency"):
        alhr.set_launch_mode(shape)
        try:
            res = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"], want_idx=True,
                               want_count=True, want_expansions=True, want_budget=True, **kw)
            torch.cuda.synchronize()
        finally:
            alhr.set_launch_mode("auto")
        for (b, h), ref in refs.items():
            compare_rows(res, ref, b, h, np.arange(1), TOL, f"768 queries {shape} d={d} {(b, h)}")


@pytest.mark.parametrize("d,bits", [(128, 64), (64, 0)])
def test_mid_size_route_predict_override(alhr, d, bits):
    """The other entry points at 768 queries (the two-warp CTA shape): alhr_predict_budget,
    alhr_route (with expansions) and alhr_forward with a budget override, against the oracle
    on sampled blocks."""
    from tree_routed_sparse_b200 import synth
    n = 2048
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(batch=96, n=n, d=d, q_start=n - 1,
                                                              score_bits=bits, seed=9)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"])
    kw = dict(q_start=wl.q_start, window=wl.window, max_keys=wl.max_keys, score_bits=bits)
    budget = alhr.predict_budget(inp["Q"], inp["K"], tree, inp["W"], **kw)
    r = alhr.route(inp["Q"], inp["K"], tree, budget, **kw)
    # an override budget of 3..96 keys, different from the predicted one
    bo = ((torch.arange(wl.bh, device="cuda", dtype=torch.int32) * 7) % 96 + 1).view(
        wl.batch, wl.heads, 1).contiguous()
    f = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, budget_override=bo, want_idx=True,
                     want_count=True, want_expansions=True, **kw)
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    rng = np.random.default_rng(4)
    for b, h in [(0, 0), (95, 7)] + [tuple(x) for x in zip(rng.integers(0, 96, 8),
                                                           rng.integers(0, 8, 8))]:
        ref = oracle_slice(cpu, wl, b, h)
        assert int(budget[b, h, 0]) == int(ref["budget"][0]), (b, h)
        compare_rows({"idx": r["idx"], "count": r["count"], "expansions": r["expansions"]},
                     ref, b, h, np.arange(1), TOL, f"route 768 d={d} {(b, h)}")
        cpu_bo = dict(cpu, W=None, budget_override=bo.cpu())
        ref_o = oracle_slice(cpu_bo, wl.replace(predictor=False), b, h)
        compare_rows(f, ref_o, b, h, np.arange(1), TOL, f"override 768 d={d} {(b, h)}")


@pytest.mark.parametrize("d,window,max_keys", [(128, 32, 50), (64, 1, 7), (64, 32, 96)])
def test_mid_size_edges_ties(alhr, d, window, max_keys):
    """The two-warp CTA shape (768 decode-style queries) with the edge settings of the small
    parity tests: window 1 or 32, a small key cap, and values in [-1, 1] so that equal scores
    are everywhere (ties to the lower start decide the sets). Sampled blocks against the oracle."""
    from tree_routed_sparse_b200 import synth
    n = 1024
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(
        batch=96, n=n, d=d, q_start=n - 1, window=window, max_keys=max_keys, qk_lo=-1, qk_hi=1,
        score_bits=0, seed=11)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"], value_bound=1)
    res = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"], q_start=wl.q_start,
                       window=window, max_keys=max_keys, value_bound=1, want_idx=True,
                       want_count=True, want_expansions=True, want_budget=True)
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    rng = np.random.default_rng(6)
    for b, h in [(0, 0), (95, 7)] + [tuple(x) for x in zip(rng.integers(0, 96, 8),
                                                           rng.integers(0, 8, 8))]:
        ref = oracle_slice(cpu, wl, b, h)
        compare_rows(res, ref, b, h, np.arange(1), TOL, f"768 ties d={d} w={window} {(b, h)}")
