"""GPU parity of the phase-2 label kernel (alhr_topk_labels, tensor-core scores + top-16 per
query) against the oracle: labels and scores bit-exact."""
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


@pytest.fixture(scope="module")
def synth():
    from tree_routed_sparse_b200 import synth as S
    return S


def _check(A, S, B, H, n, d, q_start, nq, k, lo, hi, seed, rows=None):
    K = S.uniform_int8(seed, S.TID_K, (B, H, n, d), lo, hi, "cuda")
    Q = S.uniform_int8(seed, S.TID_Q, (B, H, nq, d), lo, hi, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = A.topk_labels(Q, K, k=k, q_start=q_start, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    lab, sc = res["labels"].cpu().numpy(), res["scores"].cpu().numpy()
    Kc, Qc = K.cpu().numpy(), Q.cpu().numpy()
    for b, h in {(0, 0), (B - 1, H - 1), (B // 2, H // 2)}:
        if rows is None:
            ref_l, ref_s = orc.topk_labels(Qc[b, h], Kc[b, h], q_start, k)
            got_l, got_s = lab[b, h], sc[b, h]
        else:
            ref = [orc.topk_labels(Qc[b, h, r:r + 1], Kc[b, h], q_start + r, k) for r in rows]
            ref_l = np.concatenate([x[0] for x in ref])
            ref_s = np.concatenate([x[1] for x in ref])
            got_l, got_s = lab[b, h, rows], sc[b, h, rows]
        bad = np.nonzero((got_l != ref_l).any(1) | (got_s != ref_s).any(1))[0]
        assert len(bad) == 0, (f"b{b}h{h} rows {bad[:5].tolist()}: gpu {got_l[bad[:2]].tolist()} "
                               f"{got_s[bad[:2]].tolist()} oracle {ref_l[bad[:2]].tolist()} "
                               f"{ref_s[bad[:2]].tolist()}")


@pytest.mark.parametrize("n,d", [(64, 64), (256, 64), (2048, 64), (256, 128), (1024, 128)])
def test_labels_prefill_all_rows(alhr, synth, n, d):
    _check(alhr, synth, 2, 3, n, d, 0, n, 16, -16, 16, seed=n + d)


@pytest.mark.parametrize("n,d", [(2, 64), (8, 128), (32, 64)])
def test_labels_smallest_sequences(alhr, synth, n, d):
    """Fewer keys than a tile and than the 16 labels: short rows padded with -1."""
    _check(alhr, synth, 2, 2, n, d, 0, n, 16, -16, 16, seed=n)


@pytest.mark.parametrize("q_start,nq", [(5, 200), (1000, 24), (2047, 1), (0, 129)])
def test_labels_query_ranges(alhr, synth, q_start, nq):
    _check(alhr, synth, 2, 2, 2048, 64, q_start, nq, 16, -16, 16, seed=q_start + nq)


@pytest.mark.parametrize("k", [1, 5, 16])
def test_labels_ties_and_short_lists(alhr, synth, k):
    """Values in {-1, 0, 1}: ties everywhere, decided by the lower position."""
    _check(alhr, synth, 1, 2, 512, 128, 0, 512, k, -1, 1, seed=k)


def test_labels_extreme_values(alhr, synth):
    """The whole int8 range: scores up to 128 * 128 * 128 = 2^21 stay exact."""
    _check(alhr, synth, 1, 2, 256, 128, 0, 256, 16, -128, 127, seed=3)
    n, d = 256, 128
    K = torch.full((1, 1, n, d), -128, dtype=torch.int8, device="cuda")
    Q = torch.full((1, 1, n, d), -128, dtype=torch.int8, device="cuda")
    res = alhr.topk_labels(Q, K, k=16)
    torch.cuda.synchronize()
    assert (res["scores"][0, 0, 100] == 1 << 21).all()
    assert res["labels"][0, 0, 100].tolist() == list(range(16))


def test_labels_full_size_sampled_rows(alhr, synth):
    """The prefill workload's sizes (2 x 8 heads, N = 16384, d = 64): sampled rows."""
    rows = np.array([0, 1, 15, 16, 127, 128, 4095, 8191, 12000, 16383])
    _check(alhr, synth, 2, 8, 16384, 64, 0, 16384, 16, -16, 16, seed=11, rows=rows)


def test_labels_rejects_bad_arguments(alhr, synth):
    Q = torch.zeros((1, 1, 4, 64), dtype=torch.int8, device="cuda")
    K = torch.zeros((1, 1, 8, 64), dtype=torch.int8, device="cuda")
    for k in (0, 17):
        with pytest.raises(alhr.AlhrError):
            alhr.topk_labels(Q, K, k=k)
    with pytest.raises(alhr.AlhrError):
        alhr.topk_labels(Q, K, q_start=5)  # q_start + nq > n
