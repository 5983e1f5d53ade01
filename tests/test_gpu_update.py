"""GPU parity of the incremental tree update (alhr_update_tree) and of a decode loop built on it.

The update's contract is that the tree ends equal to a full build of the new keys, so the bar is
bit-exact against both the library's own full build (same bytes) and the oracle's tree of the
new keys (decoded from the bytes on the host). The decode loop appends one key per step, updates
the tree and routes the new query, and every step is compared with the oracle's forward over the
keys written so far."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_util import compare_rows, decode_tree, v_bits

pytestmark = pytest.mark.gpu

TOL = 1e-3
TID_NEW = 41  # stream of replacement keys (any id the workload streams do not use)


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


def _check_update(A, S, B, H, n, d, vb, lo, hi, seed):
    K_old = S.uniform_int8(seed, S.TID_K, (B, H, n, d), -vb, vb, "cuda")
    tree = A.build_tree(K_old, value_bound=vb)
    K = K_old.clone()
    if hi > lo:
        K[:, :, lo:hi] = S.uniform_int8(seed, TID_NEW, (B, H, hi - lo, d), -vb, vb, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.update_tree(K, tree, lo, hi, value_bound=vb, dev_err=err)
    full = A.build_tree(K, value_bound=vb)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(tree, full), f"update [{lo},{hi}) differs from a full build"
    # and the oracle's tree of the new keys, for two (b,h) blocks
    Kc = K.cpu().numpy()
    tc = tree.cpu().numpy()
    for b, h in {(0, 0), (B - 1, H - 1)}:
        got = decode_tree(tc[b, h], n, d, vb)
        assert np.array_equal(got, orc.build_tree(Kc[b, h])), (b, h, lo, hi)


@pytest.mark.parametrize("n,d,vb", [(1024, 64, 16), (2048, 128, 16), (4096, 128, 127),
                                    (8, 128, 16), (2, 64, 16)])
def test_update_small_ranges_equal_full_build(alhr, synth, n, d, vb):
    """Ranges of up to 64 keys (the per-ancestor delta kernel): single keys at both ends and at
    even and odd positions, pairs, a range across a 128-key chunk edge, the largest delta range."""
    ranges = [(0, 1), (n - 1, n), (n // 2, n // 2 + 1), (n // 2 - 1, n // 2), (0, 2), (1, 2)]
    if n >= 256:
        ranges += [(127, 129), (3, 67), (n - 64, n), (200, 201)]
    for k, (lo, hi) in enumerate(ranges):
        _check_update(alhr, synth, 2, 3, n, d, vb, lo, hi, seed=17 * n + d + k)


@pytest.mark.parametrize("n,d,vb", [(1024, 64, 16), (16384, 128, 16), (2048, 128, 5)])
def test_update_large_ranges_equal_full_build(alhr, synth, n, d, vb):
    """Ranges above 64 keys (chunk rebuild): 65 keys, an unaligned middle range, a tail, all."""
    for k, (lo, hi) in enumerate([(3, 68), (100, 1000), (n - 300, n), (0, n)]):
        _check_update(alhr, synth, 2, 2, n, d, vb, lo, hi, seed=31 * n + d + k)


def test_update_large_build_plan(alhr, synth):
    """A range rebuild large enough (batch * heads * keys >= 2^24) for the build's large-size
    launch plan (7 levels per streaming row group), with chunks starting mid-sequence: equal to a
    full build, and to the oracle on two blocks (copied to the host block by block)."""
    B, H, n, d, vb = 64, 8, 65536, 64, 16
    lo, hi = 1000, 41000  # 512 blocks x 40,000 keys; first rebuilt chunk starts at key 896
    need = 2 * B * H * n * d + 2 * B * H * alhr.tree_bytes(n, d, vb)
    free, _ = torch.cuda.mem_get_info()
    if need > free - (2 << 30):
        pytest.skip(f"needs {need / 2**30:.1f} GiB")
    K_old = synth.uniform_int8(3, synth.TID_K, (B, H, n, d), -vb, vb, "cuda")
    tree = alhr.build_tree(K_old, value_bound=vb)
    K = K_old.clone()
    del K_old
    K[:, :, lo:hi] = synth.uniform_int8(3, TID_NEW, (B, H, hi - lo, d), -vb, vb, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    alhr.update_tree(K, tree, lo, hi, value_bound=vb, dev_err=err)
    full = alhr.build_tree(K, value_bound=vb)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(tree, full)
    del full
    for b, h in [(0, 0), (B - 1, H - 1)]:
        got = decode_tree(tree[b, h].cpu().numpy(), n, d, vb)
        assert np.array_equal(got, orc.build_tree(K[b, h].cpu().numpy())), (b, h)
    del tree, K
    torch.cuda.empty_cache()


def test_update_empty_range_changes_nothing(alhr, synth):
    K = synth.uniform_int8(5, synth.TID_K, (1, 2, 256, 64), -16, 16, "cuda")
    tree = alhr.build_tree(K)
    before = tree.clone()
    alhr.update_tree(K, tree, 77, 77)
    torch.cuda.synchronize()
    assert torch.equal(tree, before)


def test_update_flags_keys_out_of_range(alhr, synth):
    K = synth.uniform_int8(6, synth.TID_K, (1, 1, 512, 128), -16, 16, "cuda")
    tree = alhr.build_tree(K)
    K[0, 0, 300, 5] = 40  # |key| > value_bound
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    alhr.update_tree(K, tree, 300, 301, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & alhr.DEVERR_VALUE_RANGE


@pytest.mark.parametrize("d,bits", [(128, 64), (64, 0)])
def test_decode_loop_append_update_route(alhr, synth, d, bits):
    """Keys [0, t0) present, the rest zero; each step writes key t, updates the tree over [t, t+1)
    and runs the fused forward for query t, in both launch shapes; every step equals the
    oracle's forward over the keys written so far, and the tree equals a full build."""
    B, H, n, t0, steps = 2, 2, 2048, 1500, 6
    wl = synth.WORKLOADS["decode_s64h8_n262144_d128"].replace(
        batch=B, heads=H, n=n, d=d, q_start=t0, nq=1, score_bits=bits, seed=d)
    full = synth.make_inputs(wl, "cuda")
    K_all, V = full["K"], full["V"]
    W = full["W"]
    Qs = synth.uniform_int8(wl.seed, synth.TID_Q, (B, H, steps, d), wl.qk_lo, wl.qk_hi, "cuda")
    for shape in ("latency", "throughput"):
        alhr.set_launch_mode(shape)
        try:
            K = K_all.clone()
            K[:, :, t0:] = 0
            tree = alhr.build_tree(K)
            for s in range(steps):
                t = t0 + s
                K[:, :, t] = K_all[:, :, t]
                alhr.update_tree(K, tree, t, t + 1)
                Q = Qs[:, :, s:s + 1].contiguous()
                res = alhr.forward(Q, K, V, tree, W=W, q_start=t, window=wl.window,
                                   max_keys=wl.max_keys, score_bits=bits, want_idx=True,
                                   want_count=True, want_budget=True)
                torch.cuda.synchronize()
                assert torch.equal(tree, alhr.build_tree(K)), (shape, t)
                Kc, Qc, Wc = K.cpu().numpy(), Q.cpu().numpy(), W.cpu().numpy()
                for b in range(B):
                    for h in range(H):
                        nodes = orc.build_tree(Kc[b, h])
                        ref = orc.forward(Qc[b, h], Kc[b, h], v_bits(V[b, h]), nodes, Wc, None,
                                          q_start=t, window=wl.window, max_keys=wl.max_keys)
                        compare_rows(res, ref, b, h, np.arange(1), TOL, f"{shape} t={t}")
        finally:
            alhr.set_launch_mode("auto")
