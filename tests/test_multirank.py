"""The N > 1 plumbing of bench.py on CPU: two gloo ranks.

The scan shards by (batch, head) with no data-path collective, so a
multi-GPU run is N independent copies (weak scaling) whose only collective
use is the barrier around the timed region and the max over ranks of the
measured time.  These run here without a GPU: the helpers over two spawned
gloo processes, and the reference arm under torchrun, where rank 0 alone
prints the one JSON line and the other rank exits 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    # CPU ranks even on a GPU machine (before anything initialises CUDA)
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    ws, r, _ = bench.init_dist()
    assert (ws, r) == (world, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(ws)
    out[rank] = bench.max_over_ranks(1.5 + rank, ws)
    bench.barrier(ws)
    dist.destroy_process_group()


def test_max_over_ranks_and_barrier_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
