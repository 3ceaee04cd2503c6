"""The N>1 plumbing of bench.py on CPU: two gloo ranks.

The path has no cross-GPU step (every rank is an independent replica), so the
only multi-rank logic is the reduction of the timing (max over ranks) and of
the work (sum over ranks), and the reference arm's rank-0-only rule."""
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
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r+1) ms for 10*(r+1) units
        ms, units = bench.aggregate(dist, float(rank + 1), float(10 * (rank + 1)))
        out[rank] = (ms, units)
    finally:
        dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        got = dict(out)
    # max of the times, sum of the work, the same on every rank
    assert got == {0: (2.0, 30.0), 1: (2.0, 30.0)}


def test_aggregate_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(None, 3.5, 7.0) == (3.5, 7.0)


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as the driver launches it for
    N=2: rank 0 prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--impl", "reference"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=280, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["steps"] == 1
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"] == {"value": rec["value"], "unit": rec["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
