"""The bench's multi-replica logic on CPU: two gloo ranks (no GPU).  `bench.py --gpus N` runs N
independent replicas of the layer (the single-GPU path has no exchange step); what N > 1 adds is
the barrier around the timed region, the max over ranks of the device time, the whole-job
throughput, and the reference arm running on rank 0 only."""
import json
import os
import socket
import subprocess
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
        bench.rank_barrier(world)
        # each rank's own "device time"; the job takes as long as the slowest rank
        got = bench.reduce_max(10.0 + 5.0 * rank, world, "cpu")
        out[rank] = got
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas x 4096 tokens x 10 steps in 20 ms (max over ranks) -> 4.096 M tokens/s
    assert bench.job_tokens_per_s(2, 4096, 10, 20.0) == pytest.approx(4.096e6)
    assert bench.job_tokens_per_s(1, 4096, 10, 20.0) == pytest.approx(2.048e6)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "switch_tiny", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "switch_tiny", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_cpu_baseline_repeats_a_short_sample(monkeypatch):
    """The oracle baseline repeats its sample's step (at most four times) until it has run for about
    the target time, and reports tokens over the summed time of all the repetitions."""
    sys.path.insert(0, ROOT)
    import bench
    steps = []
    monkeypatch.setattr(bench, "prepare_oracle_weights", lambda shape, inp: None)
    monkeypatch.setattr(bench, "calibrate_sample", lambda shape, inp, target: (200, 3.0))
    monkeypatch.setattr(bench, "oracle_step", lambda shape, inp, n: steps.append(n) or 3.0)
    shape = type("Shape", (), {"T": 16384})()
    out = bench.cpu_baseline(shape, None, 12.0)
    assert steps == [200] * 4
    assert out["value"] == pytest.approx(200 * 4 / 12.0)
    assert "4 float64 forward+backward steps" in out["sample"]
    steps.clear()
    monkeypatch.setattr(bench, "oracle_step", lambda shape, inp, n: steps.append(n) or 20.0)
    out = bench.cpu_baseline(shape, None, 12.0)
    assert steps == [200] and out["value"] == pytest.approx(10.0)
