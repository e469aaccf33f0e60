"""Multi-rank plumbing of bench.py on CPU: two `gloo` ranks (spawned processes).

With --gpus N every rank runs an independent replica; the job's step time is the max
over ranks, the value is N x batch tokens per that time, and the oracle reference arm
runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, loc = bench.dist_info()
        assert (w, r, loc) == (world, rank, rank)
        ms = [0.125, 0.5][rank]                   # rank 1 is the slow one
        bench.dist_barrier(world)
        mx = bench.dist_max(ms, world)
        val = bench.job_tokens_per_s(world, 8, mx)
        bench.dist_barrier(world)
        # the reference arm: ranks other than 0 leave at once (no oracle work, no output)
        rc_ref = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) \
            if rank != 0 else 0
        q.put((rank, mx, val, rc_ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, val, rc in got:
        assert mx == 0.5                          # both ranks see the slowest rank's time
        assert val == pytest.approx(2 * 8 / 0.5e-3)
        assert rc == 0


def test_single_rank_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(3.25, 1) == 3.25
    bench.dist_barrier(1)
    assert bench.job_tokens_per_s(1, 8, 1.0) == 8000.0
