"""GPU parity: the CUDA path through the C ABI against the oracle, on the same seeded inputs.

Bar: bit-exact tree sums, budgets, selected index sets, counts and expansion counts; outputs
within 1e-3 (max abs) of the oracle's fp64 attention (fp32 accumulation, bf16 V)."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_util import compare_rows, decode_tree, oracle_slice, v_bits

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


@pytest.fixture(scope="module")
def synth():
    from tree_routed_sparse_b200 import synth as S
    return S


@pytest.fixture(params=["throughput", "latency"])
def shape(request, alhr):
    """Both launch shapes of the per-query kernels on the same small inputs (the automatic choice
    would pick the latency shape for all of them)."""
    alhr.set_launch_mode(request.param)
    yield request.param
    alhr.set_launch_mode("auto")


def _to(inp, device):
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def _run_forward(A, wl, inp, **kw):
    dev = inp["Q"].device
    vb = max(-wl.qk_lo, wl.qk_hi)
    tree = A.build_tree(inp["K"], value_bound=vb)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    res = A.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"],
                    budget_override=inp["budget_override"], q_start=wl.q_start,
                    window=wl.window, max_keys=wl.max_keys, score_bits=wl.score_bits,
                    value_bound=max(-wl.qk_lo, wl.qk_hi), want_idx=True, want_count=True,
                    want_expansions=True, want_budget=True, dev_err=err, **kw)
    torch.cuda.synchronize()
    res["tree"] = tree
    res["nodes"] = A.tree_unpack(tree, wl.n, wl.d, vb)
    res["dev_err"] = int(err.item())
    return res


# ------------------------------------------------------------------ tree


@pytest.mark.parametrize("B,H,n,d", [(1, 1, 2, 64), (1, 1, 8, 128), (2, 3, 128, 64),
                                     (1, 2, 1024, 128), (2, 1, 4096, 64), (1, 1, 1 << 16, 64),
                                     (1, 3, 16, 64), (3, 1, 32, 128), (1, 1, 256, 64),
                                     (1, 5, 512, 128), (1, 3, 2048, 64)])
def test_tree_bit_exact(alhr, synth, B, H, n, d):
    """Both the library's unpack and an independent host reading of the documented layout
    give the oracle's sums."""
    K = synth.uniform_int8(7, synth.TID_K, (B, H, n, d), -16, 16, "cuda")
    tree = alhr.build_tree(K)
    nodes = alhr.tree_unpack(tree, n, d).cpu().numpy()
    tb = tree.cpu().numpy()
    Kc = K.cpu().numpy()
    for b in range(B):
        for h in range(H):
            ref = orc.build_tree(Kc[b, h])
            assert np.array_equal(nodes[b, h], ref), (b, h)
            assert np.array_equal(decode_tree(tb[b, h], n, d, 16), ref), (b, h)


@pytest.mark.parametrize("vb,n,d", [(127, 1024, 128), (1, 4096, 128), (5, 8192, 64), (16, 2048, 128)])
def test_tree_other_value_bounds(alhr, synth, vb, n, d):
    """Other bounds move the int16/int32 boundary; sums stay exact at the extremes."""
    K = synth.uniform_int8(11, synth.TID_K, (1, 2, n, d), -vb, vb, "cuda")
    K[0, 1, : n // 2] = vb
    tree = alhr.build_tree(K, value_bound=vb)
    tb = tree.cpu().numpy()
    nodes = alhr.tree_unpack(tree, n, d, vb).cpu().numpy()
    for h in range(2):
        ref = orc.build_tree(K[0, h].cpu().numpy())
        assert np.array_equal(nodes[0, h], ref)
        assert np.array_equal(decode_tree(tb[0, h], n, d, vb), ref)


def test_tree_extremes_and_range_flag(alhr):
    n, d = 2048, 128
    K = torch.full((1, 1, n, d), 16, dtype=torch.int8, device="cuda")
    K[0, 0, 1::2] = -16
    K[0, 0, :512] = 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tree = alhr.build_tree(K, dev_err=err)
    assert int(err.item()) == 0
    nodes = alhr.tree_unpack(tree, n, d)
    assert np.array_equal(nodes[0, 0].cpu().numpy(), orc.build_tree(K[0, 0].cpu().numpy()))
    K[0, 0, 77, 5] = 17
    alhr.build_tree(K, value_bound=16, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & alhr.DEVERR_VALUE_RANGE


# ------------------------------------------------------------------ fused forward, small cases


def test_forward_tiny_prefill_all_queries(alhr, synth, shape):
    """1 x 1 x 1024, d=64, fixed budget min(i+1, 32): every query against the oracle."""
    wl = synth.WORKLOADS["tiny_prefill_n1024"]
    inp = synth.make_inputs(wl, "cuda")
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    ref = oracle_slice(cpu, wl, 0, 0)
    assert np.array_equal(res["nodes"][0, 0].cpu().numpy(), ref["nodes"])
    compare_rows(res, ref, 0, 0, np.arange(wl.nq), TOL, "tiny")
    assert res["dev_err"] == 0


@pytest.mark.parametrize("n,d,w,mk,bits", [(256, 64, 16, 96, 0), (512, 128, 16, 96, 64),
                                           (1024, 64, 1, 96, 32), (512, 64, 32, 96, 0),
                                           (256, 128, 5, 7, 0), (64, 64, 16, 96, 64),
                                           (2048, 128, 16, 50, 0)])
def test_forward_predicted_budget_all_queries(alhr, synth, n, d, w, mk, bits, shape):
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(
        batch=2, heads=2, n=n, d=d, nq=n, window=w, max_keys=mk, score_bits=bits, seed=n + d + w)
    inp = synth.make_inputs(wl, "cuda")
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    for b in range(wl.batch):
        for h in range(wl.heads):
            ref = oracle_slice(cpu, wl, b, h)
            compare_rows(res, ref, b, h, np.arange(n), TOL, f"b{b}h{h}")
    assert res["dev_err"] == 0


def test_forward_ties_everywhere(alhr, synth, shape):
    """All keys equal: every candidate score ties, so only the lower-start rule decides."""
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=2, n=512, nq=512)
    inp = synth.make_inputs(wl, "cuda")
    inp["K"][:] = 3
    inp["K"][0, 1, :, ::2] = -16
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    for h in range(2):
        compare_rows(res, oracle_slice(cpu, wl, 0, h), 0, h, np.arange(512), TOL, f"h{h}")


def test_forward_extreme_values(alhr, synth, shape):
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=1, n=4096, nq=4096,
                                                       score_bits=32)
    inp = synth.make_inputs(wl, "cuda")
    inp["K"][:] = torch.where(inp["K"] >= 0, 16, -16).to(torch.int8)
    inp["Q"][:] = torch.where(inp["Q"] >= 0, 16, -16).to(torch.int8)
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    rows = np.r_[0:40, 4000:4096, np.arange(40, 4000, 37)]
    compare_rows(res, oracle_slice(cpu, wl, 0, 0, rows=rows), 0, 0, rows, TOL, "extreme")


def test_forward_budget_override_edges(alhr, synth, shape):
    """Budgets below 1 are clamped and flagged; budgets above max_keys are capped."""
    wl = synth.WORKLOADS["tiny_prefill_n1024"].replace(n=256, nq=256)
    inp = synth.make_inputs(wl, "cuda")
    bo = torch.randint(-3, 130, (1, 1, 256), dtype=torch.int32,
                       generator=torch.Generator().manual_seed(5)).to("cuda")
    inp["budget_override"] = bo
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    compare_rows(res, oracle_slice(cpu, wl, 0, 0), 0, 0, np.arange(256), TOL, "override")
    assert res["dev_err"] & alhr.DEVERR_BUDGET_LOW


def test_decode_style_queries(alhr, synth, shape):
    """q_start > 0: the last 7 positions of a 4096-key head, int64 scores, d = 128."""
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(batch=3, heads=2, n=4096,
                                                              q_start=4089, nq=7)
    inp = synth.make_inputs(wl, "cuda")
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    for b in range(3):
        for h in range(2):
            compare_rows(res, oracle_slice(cpu, wl, b, h), b, h, np.arange(7), TOL, "decode")


@pytest.mark.parametrize("n,d", [(2, 64), (4, 128), (8, 64), (16, 128)])
def test_forward_smallest_sequences(alhr, synth, n, d, shape):
    """The smallest trees (one to four levels), every query, predicted budgets."""
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=2, heads=3, n=n, d=d, nq=n,
                                                      window=2, seed=n + d)
    inp = synth.make_inputs(wl, "cuda")
    res = _run_forward(alhr, wl, inp)
    cpu = _to(inp, "cpu")
    for b in range(wl.batch):
        for h in range(wl.heads):
            compare_rows(res, oracle_slice(cpu, wl, b, h), b, h, np.arange(n), TOL, f"n={n}")
    assert res["dev_err"] == 0


# ------------------------------------------------------------------ descent variants


VARIANTS = [(True, 0), (False, 1), (False, 2), (True, 2), (False, 4), (True, 5)]


@pytest.mark.parametrize("norm,bucket", VARIANTS)
@pytest.mark.parametrize("n,d,bits", [(512, 64, 0), (1024, 128, 64)])
def test_descent_variants_all_queries(alhr, synth, norm, bucket, n, d, bits, shape):
    """Mean-normalised ranking and leaf buckets, with the predicted budget, every query."""
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(
        batch=2, heads=2, n=n, d=d, nq=n, score_bits=bits, seed=n + d + 10 * bucket + norm)
    inp = synth.make_inputs(wl, "cuda")
    res = _run_forward(alhr, wl, inp, score_norm=norm, bucket_log=bucket)
    cpu = _to(inp, "cpu")
    for b in range(wl.batch):
        for h in range(wl.heads):
            ref = oracle_slice(cpu, wl, b, h, score_norm=norm, bucket_log=bucket)
            compare_rows(res, ref, b, h, np.arange(n), TOL, f"norm={norm} b={bucket} b{b}h{h}")
    assert res["dev_err"] == 0


@pytest.mark.parametrize("norm,bucket", [(False, 2), (True, 3), (True, 0)])
def test_descent_variants_route_and_ties(alhr, synth, norm, bucket, shape):
    """The route entry point with a budget override (values in {-1, 0, 1}: ties everywhere),
    against the oracle and against the fused forward."""
    wl = synth.WORKLOADS["tiny_prefill_n1024"].replace(n=512, nq=512, qk_lo=-1, qk_hi=1,
                                                       seed=77 + bucket)
    inp = synth.make_inputs(wl, "cuda")
    vb = 1
    tree = alhr.build_tree(inp["K"], value_bound=vb)
    kw = dict(q_start=0, window=wl.window, max_keys=wl.max_keys, value_bound=vb,
              score_norm=norm, bucket_log=bucket)
    budget = inp["budget_override"]
    r = alhr.route(inp["Q"], inp["K"], tree, budget, **kw)
    f = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, budget_override=budget, want_idx=True,
                     want_count=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(r["idx"], f["idx"]) and torch.equal(r["count"], f["count"])
    cpu = _to(inp, "cpu")
    for b in range(wl.batch):
        for h in range(wl.heads):
            ref = oracle_slice(cpu, wl, b, h, score_norm=norm, bucket_log=bucket)
            compare_rows({"idx": r["idx"], "count": r["count"], "out": f["out"]}, ref, b, h,
                         np.arange(wl.nq), TOL, f"route norm={norm} b={bucket}")


# ------------------------------------------------------------------ unfused entry points


@pytest.mark.parametrize("d,bits", [(64, 0), (128, 64)])
def test_unfused_path_matches_oracle_and_fused(alhr, synth, d, bits, shape):
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=3, n=1024, nq=1024, d=d,
                                                       score_bits=bits)
    inp = synth.make_inputs(wl, "cuda")
    fused = _run_forward(alhr, wl, inp)
    kw = dict(q_start=0, window=wl.window, max_keys=wl.max_keys, score_bits=bits)
    budget = alhr.predict_budget(inp["Q"], inp["K"], fused["tree"], inp["W"], **kw)
    routed = alhr.route(inp["Q"], inp["K"], fused["tree"], budget, **kw)
    out = alhr.attend(inp["Q"], inp["K"], inp["V"], routed["idx"], routed["count"],
                      q_start=0, window=wl.window, max_keys=wl.max_keys)
    torch.cuda.synchronize()
    assert torch.equal(budget, fused["budget"])
    assert torch.equal(routed["idx"], fused["idx"])
    assert torch.equal(routed["count"], fused["count"])
    assert torch.equal(routed["expansions"], fused["expansions"])
    cpu = _to(inp, "cpu")
    unf = dict(out=out.cpu(), idx=routed["idx"].cpu(), count=routed["count"].cpu(),
               expansions=routed["expansions"].cpu(), budget=budget.cpu())
    for h in range(3):
        compare_rows(unf, oracle_slice(cpu, wl, 0, h), 0, h, np.arange(1024), TOL, f"h{h}")


def test_attend_skips_bad_indices(alhr, synth):
    wl = synth.WORKLOADS["tiny_prefill_n1024"].replace(n=64, nq=64)
    inp = synth.make_inputs(wl, "cuda")
    idx = torch.full((1, 1, 64, 96), -1, dtype=torch.int32, device="cuda")
    count = torch.full((1, 1, 64), 3, dtype=torch.int32, device="cuda")
    pos = torch.arange(64, device="cuda", dtype=torch.int32)
    idx[0, 0, :, 0] = pos
    idx[0, 0, :, 1] = pos + 1          # the future key: skipped
    idx[0, 0, :, 2] = pos // 2
    count[0, 0, 0] = 0                 # empty selection: a zero row
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = alhr.attend(inp["Q"], inp["K"], inp["V"], idx, count, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & alhr.DEVERR_INDEX
    Q, K = (inp[k][0, 0].cpu().numpy() for k in "QK")
    Vb = v_bits(inp["V"][0, 0])
    o = out[0, 0].cpu().numpy()
    assert np.all(o[0] == 0)
    for i in range(1, 64):
        sel = np.unique(np.array([i, i // 2], dtype=np.int32))
        ref = orc.attend(Q[i], K, Vb, sel)
        assert np.abs(o[i] - ref).max() <= TOL


def test_empty_and_invalid_calls(alhr, synth):
    wl = synth.WORKLOADS["tiny_prefill_n1024"].replace(n=64, nq=0)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"])
    res = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, budget_override=inp["budget_override"])
    assert res["out"].numel() == 0
    with pytest.raises(alhr.AlhrError):
        alhr.forward(inp["Q"], inp["K"], inp["V"], tree, window=33,
                     budget_override=inp["budget_override"])
