"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun
launches them.  Each GPU rank runs an independent replica (the linear has no
exchange step), so what the ranks share is the timing: the job's time is the
slowest rank's (max over ranks) and its throughput is the units all ranks
processed over that time, and every rank replays the timed region the same
number of times.  The reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank device times (ms): rank 1 is the slower one in the first
        # entry, rank 0 in the second
        mine = [10.0 + 5.0 * rank, 7.0 - 2.0 * rank]
        got = bench.max_over_ranks(mine, world, "cpu")
        # the replay count follows the slowest rank's first replay
        reps = bench.agreed_replays(bench.MIN_TIMED_MS / (10.0 + 10.0 * rank), world, "cpu")
        torch.distributed.barrier()

        class A:
            workload = "single_linear_m32"
            steps = 1
            warmup = 1

        ref = bench.run_reference(A, rank, world) if rank != 0 else "rank 0 not run here"
        q.put((rank, got, ref, reps))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_time_and_reference_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in procs:
        rank, got, ref, reps = q.get(timeout=120)
        out[rank] = (got, ref, reps)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time for every entry
    assert out[0][0] == out[1][0] == [15.0, 7.0]
    # the reference arm does no work on the other ranks
    assert out[1][1] is None
    # both ranks replay the timed region equally often: enough for the slower
    # rank (first replay MIN_TIMED_MS / 10 on rank 0, MIN_TIMED_MS / 20 on rank 1)
    assert out[0][2] == out[1][2] == 10


def test_job_throughput_is_all_ranks_units_over_max_time():
    import bench

    # 512 tokens per rank and step, 10 steps, 2 ranks, slowest rank 40 ms
    assert bench.job_throughput(512, 10, 2, 40.0) == pytest.approx(512 * 10 * 2 / 0.040)
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
