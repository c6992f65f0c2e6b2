"""The benchmark's multi-rank logic on CPU (gloo, world size 2).

On N GPUs the benchmark runs one process per GPU: every rank processes the same
units (weak scaling), the timing is the slowest rank's, and the job throughput is
the units of all ranks over that time; the reference arm runs on rank 0 alone.
These tests run that logic with two CPU processes: the all-reduce MAX of the
timings over a gloo process group, the throughput aggregation, and the reference
arm under torch.distributed.run."""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_seconds = 1.5 if rank == 1 else 0.5          # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_seconds, world, "cpu")
        dist.barrier()
        value = bench.job_throughput(1000.0, world, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_slowest_rank_and_job_throughput_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["slowest"] == 1.5                          # every rank sees the slowest time
        assert r["value"] == pytest.approx(2 * 1000.0 / 1.5)  # units of both ranks / slowest time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(0.25, 1, "cpu") == 0.25
    assert bench.job_throughput(10.0, 1, 2.0) == 5.0


def test_reference_arm_runs_on_rank_zero_only():
    """`bench.py --impl reference` under torch.distributed.run with two processes: rank 0
    prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "single_head_d128_n4096",
           "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.2"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
