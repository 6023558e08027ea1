"""The benchmark's multi-rank plumbing on CPU with world size 2 (gloo): the
max-over-ranks timing reduction, the whole-job throughput, per-rank input
replicas, and the reference arm under torchrun (rank 0 prints, rank 1 exits 0).
The layer itself shards by tokens with no exchange, so this is all the
multi-GPU path has besides the per-rank kernels."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r reports (r + 1, 10 - r): the maxima are (world, 10)
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], "cpu")
        # each replica draws its own synthetic inputs (the benchmark passes
        # seed_tag = rank), here at a small size of the same generator
        from quantized_gemm_column_b200 import inputs
        X, _, _ = inputs.workload1(l=256, m=128, n=256, seed_tag=rank)
        sample = inputs.bf16_as_f32(X)[0, :8]
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "sample": sample.tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    outs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for o in outs:
        assert o["max"] == [2.0, 10.0]
    # replicas do not share inputs
    assert not np.allclose(outs[0]["sample"], outs[1]["sample"])


def test_max_over_ranks_single_process():
    import bench
    assert bench.max_over_ranks([3.0, 1.5], "cpu") == [3.0, 1.5]


def test_job_value_is_whole_job():
    import bench
    # 2 ranks, each 1 TFLOP per step in 1 ms -> 2000 TFLOP/s for the job
    assert bench.job_value(1e12, 2, 1.0) == pytest.approx(2000.0)
    assert bench.job_value(1e12, 1, 1.0) == pytest.approx(1000.0)


@pytest.mark.slow
def test_reference_arm_under_torchrun(tmp_path):
    """`bench.py --impl reference` as the driver launches it for N = 2: one
    JSON line from rank 0 with impl "reference", exit status 0 on both ranks."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_measured_traffic_follows_kernel_sources(tmp_path, monkeypatch):
    """The roofline's DRAM traffic comes from the committed ncu capture
    (a JSON record) only while the kernel sources hash to the digest it
    records."""
    import bench
    prof = tmp_path / "traffic.json"
    prof.write_text(json.dumps({"digest": bench.kernel_digest(), "bytes_per_step": {"split-quant": 123}}))
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(prof))
    assert bench.measured_traffic("split-quant") == 123
    assert bench.measured_traffic("gemm") is None
    prof.write_text(json.dumps({"digest": "0000000000000000", "bytes_per_step": {"split-quant": 123}}))
    assert bench.measured_traffic("split-quant") is None
    prof.write_text("not json")
    assert bench.measured_traffic("split-quant") is None


def test_reference_arm_stops_at_its_time_budget(monkeypatch, capsys):
    """The oracle arm times at most its wall-clock budget of steps, whatever
    step count it is given, and says how many it timed beside the request;
    its config is the GPU arm's workload."""
    import argparse
    import bench
    monkeypatch.setattr(bench, "REF_WARMUP_S", 0.05)
    monkeypatch.setattr(bench, "REF_TIMED_S", 0.2)
    args = argparse.Namespace(gpus=1, steps=10**6, warmup=10**6)
    bench.run_reference(args, 0, 1)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert 1 <= d["steps"] < d["steps_requested"] == 10**6
    assert 1 <= d["warmup"] < d["warmup_requested"] == 10**6
    assert d["config"]["workload"] == bench.WORKLOAD
    assert (d["config"]["l"], d["config"]["m"], d["config"]["n"]) == (bench.L, bench.M, bench.N)
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
