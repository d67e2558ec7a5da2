"""The multi-process path of bench.py on CPU (gloo, world size 2): process-group set-up, the
max-over-ranks reduction and barrier the timed region uses, and the reference arm under
torchrun, where rank 0 alone runs the oracle and prints one JSON line and the other rank
exits 0 without work. (The path shards into independent replicas; there is no data-path
collective to test.)"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# with CUDA visible, bench.py takes NCCL and one GPU per rank
pytestmark = pytest.mark.skipif(torch.cuda.is_available() and torch.cuda.device_count() < 2,
                                reason="two ranks need two GPUs when CUDA is visible")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    out[rank] = bench.max_over_ranks(1.5 + rank, w)   # each rank's "time"; the max wins
    bench.barrier(w)
    dist.destroy_process_group()


def test_dist_setup_and_max_over_ranks_gloo():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:      # no fork of a threaded process
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    sys.path.insert(0, ROOT)
    import bench
    # the config both arms print is the workload's name and sizes, nothing else
    assert d["config"] == bench.config_of("prefill_gqa_n32768")
