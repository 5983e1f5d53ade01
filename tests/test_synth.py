"""The seeded input generator: SplitMix64 known answers, device-independent bits, slices."""
import numpy as np
import torch

from tree_routed_sparse_b200 import synth


def test_splitmix64_published_sequence():
    # first outputs of splitmix64 started from state 0 (Vigna's reference implementation)
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    got = [synth.mix64(k * synth.GAMMA) for k in (1, 2, 3)]
    assert got == expect


def test_torch_words_match_python_ints():
    for seed, tid in [(0, 1), (3, 2), (123, 6)]:
        base = synth.stream_base(seed, tid)
        start = 1_000_003
        words = synth.raw_words(seed, tid, start, 64, "cpu").numpy().view(np.uint64)
        ref = [synth.mix64(base + (start + k + 1) * synth.GAMMA) for k in range(64)]
        assert [int(x) for x in words] == ref


def test_uniform_int8_range_and_slices():
    x = synth.uniform_int8(0, synth.TID_K, (4, 100_000), -16, 16)
    assert x.dtype == torch.int8 and int(x.min()) == -16 and int(x.max()) == 16
    counts = torch.bincount((x.flatten().to(torch.int64) + 16), minlength=33).float()
    assert (counts / counts.mean() - 1).abs().max() < 0.05  # ~12000 per bin, 5 sigma
    part = synth.uniform_int8(0, synth.TID_K, (2, 100_000), -16, 16, offset=200_000)
    assert torch.equal(part, x[2:])
    assert torch.equal(x, synth.uniform_int8(0, synth.TID_K, (4, 100_000), -16, 16))


def test_normal_bf16_moments():
    v = synth.normal_bf16(0, synth.TID_V, (200_000,)).float()
    assert abs(float(v.mean())) < 0.01 and abs(float(v.std()) - 1) < 0.01


def test_workload_inputs_shapes():
    wl = synth.WORKLOADS["tiny_prefill_n1024"]
    inp = synth.make_inputs(wl)
    assert inp["Q"].shape == (1, 1, 1024, 64) and inp["V"].dtype == torch.bfloat16
    assert inp["W"] is None
    b = inp["budget_override"][0, 0]
    assert b[:3].tolist() == [1, 2, 3] and int(b[31]) == 32 and int(b.max()) == 32
    wl2 = synth.WORKLOADS["prefill_b4h8_n4096"]
    small = wl2.replace(batch=1, heads=2, n=256, nq=256)
    inp2 = synth.make_inputs(small)
    assert inp2["W"].shape == (32, 128) and int(inp2["W"].abs().max()) <= 4


def test_recall_planting():
    wl = synth.WORKLOADS["recall_b2h4_n16384_d128"].replace(n=1024, nq=1024, plant_pairs=16)
    inp = synth.make_inputs(wl)
    for b in range(wl.batch):
        p, u = synth.plant_positions(wl, b)
        assert len(set(p.tolist())) == 16 and len(set(u.tolist())) == 16
        assert int(p.max()) < 512 and int(u.min()) >= 512
        diff = inp["Q"][b][:, u].to(torch.int16) - inp["K"][b][:, p].to(torch.int16)
        assert int(diff.abs().max()) <= 2


def test_block_inputs_are_slices_of_the_batch():
    wl = synth.WORKLOADS["recall_b2h4_n16384_d128"].replace(n=256, nq=256, plant_pairs=8)
    full = synth.make_inputs(wl)
    for lo, hi in [(0, 8), (1, 6), (3, 4), (4, 8), (5, 5)]:
        part = synth.make_block_inputs(wl, lo, hi)
        for k in ("Q", "K", "V"):
            flat = full[k].reshape(-1, *full[k].shape[2:])
            assert torch.equal(part[k][0], flat[lo:hi]), (lo, hi, k)
        assert torch.equal(part["W"], full["W"])


def test_shards_of_a_global_batch():
    from tree_routed_sparse_b200 import shard
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=3, n=128, nq=128)
    g = shard.global_workload(wl, 2)
    assert g.batch == 2 and g.bh == 6
    full = synth.make_inputs(g)
    parts = [shard.shard_inputs(g, 2, r) for r in range(2)]
    assert [(lo, hi) for lo, hi, _ in parts] == [(0, 3), (3, 6)]
    for r, (lo, hi, inp) in enumerate(parts):
        assert inp["Q"].shape == (1, 3, 128, 64)
        assert torch.equal(inp["K"], full["K"][r:r + 1]) and torch.equal(inp["Q"], full["Q"][r:r + 1])
    lo, hi, inp = shard.shard_inputs(g, 4, 1)  # blocks [2, 4): not whole sequences
    assert (lo, hi) == (2, 4) and inp["K"].shape == (1, 2, 128, 64)
    assert torch.equal(inp["K"][0], full["K"].reshape(6, 128, 64)[2:4])


def test_live_classes_zero_the_upper_predictor_rows():
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=1, n=64, nq=64,
                                                        live_classes=20)
    W = synth.make_inputs(wl)["W"]
    assert int(W[20:].abs().max()) == 0 and int(W[:20].abs().max()) > 0
