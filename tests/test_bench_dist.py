"""The multi-process path of bench.py on CPU (gloo, world size 2).

The grouped linear hot path has no exchange step, so ``bench.py --gpus N``
runs N independent replicas; the only cross-rank work is the barrier and the
max-over-ranks reduction of each timed region, and the job's throughput
counts every replica's flops over the slowest rank's time.  The reference arm
(the oracle on the host) runs on rank 0 alone and prints one line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    assert out[0] == out[1] == 15.0


def test_single_process_and_job_throughput():
    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    # two replicas, 1 TFLOP each per step, slowest rank 2 ms per step
    assert bench.job_tflops(1e12, 2, 2.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_prints_once():
    """Rank 0 runs the oracle sample and prints one JSON line; rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    # the line carries the same contract keys as the GPU arm's
    for k in ("metric", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "dtype", "data",
              "config", "e2e", "cpu_baseline"):
        assert k in d, k
    assert d["higher_is_better"] is True and d["config"]["workload"].startswith("bf16_g8")
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["sample"]
