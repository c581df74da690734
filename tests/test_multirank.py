"""The benchmark's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1 (no GPU).

Each rank of a multi-GPU run times its own batch; the job's step time is the max over ranks and
the job's throughput counts every rank's tokens. The reference arm runs on rank 0 only.
"""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # per-rank timings that differ in every position: the max must pick each one's slowest
        ms = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.5 * (rank + 1)], dist)
        q.put((rank, ms, bench.job_throughput(world, 131072, ms[0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r for r, _, _ in res] == [0, 1]
    for _, ms, value in res:
        assert ms == [2.0, 5.0, 1.0]
        assert value == pytest.approx(2 * 131072 / 2.0e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]
    assert bench.job_throughput(1, 131072, 1.0) == pytest.approx(131072e3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    bench.run_reference(None, rank=1)  # other ranks exit before reading any argument
    assert capsys.readouterr().out == ""
