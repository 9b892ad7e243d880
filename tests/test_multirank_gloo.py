"""The multi-GPU (N > 1) host path of bench.py on CPU: two ranks over a
gloo process group check that every rank draws its own batch, that the
timings are reduced as the maximum over ranks, and that the job value
counts every rank's bytes over the slowest rank's time.  The reference
arm under torchrun prints one line, from rank 0 only."""
import datetime
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        w, r, _ = bench.dist_env()
        cpu = torch.device("cpu")
        my_ms = 10.0 * (r + 1)                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(my_ms, w, cpu)
        ranks = bench.sum_over_ranks(1.0, w, cpu)
        b = workloads.make_batch("prefill", bench.rank_seed(r), T=64, H=128)
        digest = int(b.idx.sum()) * 1000003 + int(b.x.view(torch.int16).sum())
        bench.barrier(w)
        out[r] = (w, slowest, ranks, digest,
                  bench.job_value(1000, 5, w, slowest))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_shard():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 2
    assert r0[1] == r1[1] == 20.0                    # max over ranks
    assert r0[2] == r1[2] == 2.0
    assert r0[3] != r1[3]                            # independent batches
    # 2 ranks x 1000 bytes x 5 steps over 20 ms
    assert r0[4] == pytest.approx(2 * 1000 * 5 / 0.020 / 1e9)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
    # the same workload as the GPU arm: the whole prefill batch per step
    assert rec["config"]["T"] == 4096 and rec["config"]["bytes_per_step"] > 1e9
