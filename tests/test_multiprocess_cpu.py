"""The multi-GPU mode of bench.py is independent replicas (the path has no exchange
step): each rank times its own steps, the job time is the max over ranks and the work is
the sum.  Checked here with two gloo ranks on the CPU, and the reference arm's rule that
only rank 0 works and prints."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    ms, units = bench.aggregate(10.0 + 5.0 * rank, 100.0 * (rank + 1), dist, "cpu")
    q.put((rank, ms, units))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, units in got:
        assert ms == 15.0          # the slower rank decides the job time
        assert units == 300.0      # both ranks' work counts


def test_aggregate_single_process():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.aggregate(3.0, 7.0) == (3.0, 7.0)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--cpu-seconds", "0.1"], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0
    assert out.stdout.strip() == ""


def test_reference_arm_rank0_json_line():
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--cpu-seconds", "0.2"], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_backward_workload():
    """The oracle arm of `--workload backward`: one JSON line in TFLOP/s with the workload
    string the GPU arm prints for the same token batch."""
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "backward", "--backward-batch", "1024", "--cpu-seconds", "0.1"], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["config"]["workload"] == "factor and scale gradients, 11008x4096 r=2432 layer, 1024 tokens"
    assert rec["cpu_baseline"]["kind"] == "oracle"
