"""The multi-rank side of bench.py on the CPU: two gloo ranks (no GPU).

bench.py runs one independent stack per GPU rank (replicas: the layers of a
step are sharded across ranks with no data-path collective), takes every
device time as the slowest rank's, and reports the whole job's layers per
time.  These tests run its rank reduction over gloo with world size 2 and its
reference arm under torch.distributed.run with two ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _reduce_worker(rank, world, port, values, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(values[rank], torch.device("cpu"))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    values = [[1.5, 7.0, 0.25], [2.5, 3.0, 0.5]]
    mp.start_processes(_reduce_worker, args=(2, _free_port(), values, str(tmp_path)), nprocs=2,
                       join=True, start_method="spawn")
    want = [max(a, b) for a, b in zip(*values)]
    for r in range(2):
        with open(tmp_path / f"r{r}.json") as f:
            assert json.load(f) == want


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 1.0], torch.device("cpu")) == [3.0, 1.0]


def test_job_value_counts_every_rank_layers():
    # 2 ranks x 1000 layers in the slowest rank's 2 ms: 1 us per layer of the job
    assert bench.job_us_per_layer(2.0, 1000, 2) == pytest.approx(1.0)
    assert bench.job_us_per_layer(2.0, 1000, 1) == pytest.approx(2.0)


def test_reference_arm_under_two_ranks():
    """Rank 0 alone runs the CPU oracle and prints one JSON line; rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "7b_attn_0.1bpw_residual"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "us/layer"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
