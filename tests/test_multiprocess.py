"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduction, per-rank batches for weak scaling, and the
reference arm printing exactly one line from rank 0 under torchrun."""
from __future__ import annotations

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


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [3.5, 7.25][rank]
    got = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
    with open(f"{out_path}.{rank}", "w") as f:
        f.write(repr(got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    port = free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path / "r")), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        assert float(open(tmp_path / f"r.{r}").read()) == 7.25


def test_rank_batches_are_independent_and_same_shape():
    sys.path.insert(0, ROOT)
    import bench

    xs0, ps0 = bench.rank_inputs(0)
    xs1, ps1 = bench.rank_inputs(1)
    for a, b, pa, pb in zip(xs0, xs1, ps0, ps1):
        assert a.shape == b.shape and a.dtype == b.dtype
        assert not np.array_equal(a[:4], b[:4])
        assert np.array_equal(pa, pb)


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["cpu_baseline"]["kind"] == "oracle"
    # the contract's keys: the same metric, unit and workload as the device arm, an oracle
    # cpu_baseline describing the run, and an e2e with no host-device traffic
    sys.path.insert(0, ROOT)
    import bench

    assert rec["config"]["workload"] == bench.FLUX_WORKLOAD
    assert rec["unit"] == "GB/s" and rec["higher_is_better"] is True and rec["value"] > 0
    cb = rec["cpu_baseline"]
    assert cb["value"] == rec["value"] and cb["cores"] >= 1 and cb["sample"]
    assert rec["e2e"] == {"value": rec["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
