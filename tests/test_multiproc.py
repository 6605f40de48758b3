"""The multi-process plumbing of bench.py on CPU: two ranks over gloo, as the
benchmark runs under torchrun with one process per GPU.  Checks the
rendezvous, the max-over-ranks timing, the barrier, the whole-job rate and
that only rank 0 runs the CPU reference arm."""
import multiprocessing as mp
import os
import socket

import pytest

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    try:
        w, r, local = bench.dist_setup(None)
        # each rank times its own replica; the job takes the slowest rank's times
        mine = [10.0 + rank, 5.0 - rank, 100.0 * (rank + 1)]
        got = bench.reduce_max(mine, w)
        bench.barrier(w)
        out.put((r, w, local, dist.get_backend(), got))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    port = _free_port()
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in results] == [0, 1]
    for rank, world, local, backend, got in results:
        assert world == 2 and local == rank and backend == "gloo"
        assert got == [11.0, 5.0, 200.0]


def test_job_rate_counts_every_rank_over_the_slowest():
    # two replicas of 2e12 FLOP per step, 10 steps, slowest rank 20 ms
    assert bench.job_rate(2, 2e12, 10, 20.0) == pytest.approx(2e15)
    assert bench.job_rate(1, 2e12, 10, 20.0) == pytest.approx(1e15)


def test_reference_arm_runs_on_rank_zero_only():
    # under torchrun every rank but 0 leaves the CPU reference arm at once
    assert bench.run_reference(None, 2, 1) is None


def test_single_process_needs_no_process_group():
    for key in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(key, None)
    assert bench.dist_setup(None) == (1, 0, 0)
    assert bench.reduce_max([1.0, 2.0], 1) == [1.0, 2.0]
