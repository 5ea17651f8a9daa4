"""The N > 1 path of bench.py on CPU: two gloo ranks (127.0.0.1).

The layer is one GPU's work, so N GPUs run N replicas with no collective on
the data path; the only cross-rank step is the timing: the slowest rank's
time, and the whole job's work over it.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_ms)
        value = bench.whole_job_tflops(2.0e12, 4, world, slowest)
        out[rank] = (slowest, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_two_gloo_ranks():
    world = 2
    port = _free_port()
    # spawn, not fork: the test process may already run OpenMP threads
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        slowest, value = res[rank]
        assert slowest == 15.0                       # both ranks see the max
        # 2 ranks x 4 steps x 2e12 flops over 15 ms
        assert value == pytest.approx(2 * 4 * 2.0e12 / 15e-3 / 1e12)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.whole_job_tflops(1e12, 10, 1, 100.0) == pytest.approx(100.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    """Under torchrun only rank 0 runs and prints the reference line."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args: called.append(1) or {})
    assert bench.main() == 0
    assert called == [] and capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the oracle on the host cores) on the tiny
    workload: one JSON line with the contract's keys."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT,
                         env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_step_stats():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.step_stats([]) is None
    one = bench.step_stats([0.1])
    assert one == {"median_us": 100.0, "p10_us": 100.0, "p90_us": 100.0}
    st = bench.step_stats([0.1 + 0.001 * i for i in range(50)])   # 100 .. 149 µs
    assert st["median_us"] == pytest.approx(124.5)
    assert 100.0 <= st["p10_us"] < st["median_us"] < st["p90_us"] <= 149.0


def test_stack_shape_counts():
    import bench
    counts = bench.stack_shape_counts()
    assert sum(counts.values()) == 152
    assert counts == {(3072, 9216): 19, (3072, 3072): 19, (3072, 12288): 19, (12288, 3072): 19,
                      (3072, 21504): 38, (15360, 3072): 38}
