"""bench.py's reference arm (the oracle on the host cores) keeps the bench line's contract:
one JSON line on rank 0 with the metric, a positive value, the CPU-baseline description and an
e2e entry without copies; other ranks print nothing and exit 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env):
    env = dict(os.environ, **extra_env)
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
           "--warmup", "0", "--workload", "tiny_prefill_n1024", "--row-stride", "256"]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_bench_line():
    p = _run({})
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "queries/s"
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "tiny_prefill_n1024" in d["config"]["workload"]


def test_reference_arm_other_ranks_stay_silent():
    p = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [l for l in p.stdout.splitlines() if l.startswith("{")]


def test_reference_steps_are_timed_not_scaled():
    """Each reference step is the listed rows of every block, fully computed: the queries per
    step times the steps equal the queries the oracle computed, and ms_per_step x steps is the
    measured time (it fits in the process's own run time)."""
    import time
    t0 = time.perf_counter()
    env = dict(os.environ)
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
           "--warmup", "1", "--workload", "tiny_prefill_n1024", "--row-stride", "64"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    wall = time.perf_counter() - t0
    assert p.returncode == 0, p.stderr[-2000:]
    d = json.loads([l for l in p.stdout.splitlines() if l.startswith("{")][0])
    assert d["queries_per_step"] == 1024 // 64
    assert d["ms_per_step"] * d["steps"] / 1e3 < wall
    # value = queries / summed step time
    assert abs(d["value"] - d["queries_per_step"] / (d["ms_per_step"] / 1e3)) < 1e-6 * d["value"]
    assert "no scaling" in d["cpu_baseline"]["sample"]


def test_oracle_steps_cover_every_row_once():
    sys.path.insert(0, ROOT)
    import bench
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS["prefill_b4h8_n4096"].replace(batch=1, heads=2, n=64, nq=64)
    inp = synth.make_inputs(wl, "cpu")
    r = bench.oracle_steps(wl, inp, steps=8, row_stride=8)
    assert r["queries"] == 2 * 64 and len(r["step_s"]) == 8 and r["value"] > 0
    st = bench.oracle_single_thread(wl, inp)
    assert st["cores"] == 1 and st["block_s"] > 0 and st["value"] == 64 / st["block_s"]


def test_gpus_flag_relaunches_under_torchrun():
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.torchrun_command(["--gpus", "8", "--steps", "20"], 8, 29511)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=8" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29511" in cmd
    assert cmd[-4:] == ["--gpus", "8", "--steps", "20"] and cmd[-5].endswith("bench.py")


def test_world_size_must_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import pytest
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(4)
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.dist_setup(1) == (None, 0, 1)


def test_gpus_without_devices_fails_loudly():
    """--gpus 2 with no CUDA device: an error, never a silent one-GPU number."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1"]
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK")}
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode != 0
    assert not [l for l in p.stdout.splitlines() if l.startswith("{")]


def test_both_arms_share_config():
    sys.path.insert(0, ROOT)
    import bench
    from tree_routed_sparse_b200 import synth
    wl = synth.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert bench.bench_config(wl)["workload"].startswith("prefill_b2h8_n16384: batch 2, heads 8")
