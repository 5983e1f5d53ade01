"""The overlapped host pipeline returns, for every batch, exactly what the direct calls return."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("buffers", [2, 1])
def test_pipeline_matches_direct_calls(buffers):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_routed_sparse_b200 import alhr, build, synth
    from tree_routed_sparse_b200.pipeline import HostPipeline
    build.build()
    base = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=2, heads=2, n=1024, nq=1024)
    batches = [synth.make_inputs(base.replace(seed=s), "cpu") for s in range(5)]
    hosts = [{k: (None if v is None else v.pin_memory()) for k, v in b.items()} for b in batches]
    outs = [torch.empty((2, 2, 1024, 64), dtype=torch.float32).pin_memory() for _ in batches]
    kw = dict(q_start=0, window=base.window, max_keys=base.max_keys, score_bits=0, value_bound=16)
    pipe = HostPipeline(hosts[0], buffers=buffers, **kw)
    for h, o in zip(hosts, outs):
        pipe.submit(h, o)
    pipe.synchronize()
    for b, o in zip(batches, outs):
        d = {k: (None if v is None else v.cuda()) for k, v in b.items()}
        tree = alhr.build_tree(d["K"])
        ref = alhr.forward(d["Q"], d["K"], d["V"], tree, W=d["W"], **kw)["out"]
        torch.cuda.synchronize()
        assert torch.equal(o, ref.cpu())
