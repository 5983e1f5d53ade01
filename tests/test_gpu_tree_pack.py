"""alhr_tree_pack: plain int32 node rows into the library's tree layout (the inverse of
alhr_tree_unpack), checked against the oracle's tree and against alhr_build_tree."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc

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


@pytest.mark.parametrize("n,d,vb", [(1024, 64, 16), (4096, 128, 16), (512, 128, 127), (2, 128, 16)])
def test_pack_of_oracle_nodes_equals_build(alhr, n, d, vb):
    from tree_routed_sparse_b200 import synth
    K = synth.uniform_int8(7, synth.TID_K, (2, 3, n, d), -vb, vb, "cuda")
    Kc = K.cpu().numpy()
    nodes = torch.from_numpy(np.stack([np.stack([orc.build_tree(Kc[b, h]) for h in range(3)])
                                       for b in range(2)])).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = alhr.tree_pack(nodes, value_bound=vb, dev_err=err)
    built = alhr.build_tree(K, value_bound=vb)
    torch.cuda.synchronize()
    assert torch.equal(packed, built)
    assert torch.equal(alhr.tree_unpack(packed, n, d, vb), nodes)
    assert int(err.item()) == 0


def test_route_on_a_packed_tree(alhr):
    """A caller holding int32 node rows routes with them through the pack."""
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS["recall_b2h4_n16384_d128"].replace(batch=1, heads=2, n=2048, nq=2048,
                                                            plant_pairs=0)
    inp = synth.make_inputs(wl, "cuda")
    tree = alhr.build_tree(inp["K"])
    nodes = alhr.tree_unpack(tree, wl.n, wl.d)
    tree2 = alhr.tree_pack(nodes)
    kw = dict(window=16, max_keys=96, score_bits=64)
    a = alhr.forward(inp["Q"], inp["K"], inp["V"], tree, W=inp["W"], want_idx=True, **kw)
    b = alhr.forward(inp["Q"], inp["K"], inp["V"], tree2, W=inp["W"], want_idx=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(a["idx"], b["idx"]) and torch.equal(a["out"], b["out"])


def test_out_of_range_narrow_value_is_flagged(alhr):
    """A value no sum of keys within the bound can take on an int16 level: flagged, saturated."""
    n, d = 64, 128
    nodes = torch.zeros((1, 1, n - 1, d), dtype=torch.int32, device="cuda")
    nodes[0, 0, 0, 5] = 40000  # level 1: |sum of two keys| <= 32
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tree = alhr.tree_pack(nodes, dev_err=err)
    back = alhr.tree_unpack(tree, n, d)
    torch.cuda.synchronize()
    assert int(err.item()) == 0x2
    assert int(back[0, 0, 0, 5]) == 32767
    nodes[0, 0, 0, 5] = 33  # within int16 but above 16 * 2: still not a sum of in-bound keys
    err.zero_()
    alhr.tree_pack(nodes, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0x2
