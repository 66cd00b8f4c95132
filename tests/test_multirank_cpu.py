"""Host logic of the N > 1 bench path as two gloo ranks on the CPU: the timed region is reduced with
MAX over ranks and the whole-job throughput counts every rank's tokens over that time (replicas,
no data-path collective)."""
import datetime
import os
import socket
from types import SimpleNamespace

import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as td
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        got = bench.max_over_ranks(ms, "cpu")
        q.put((rank, got, bench.job_throughput(world, 100, got)))
        td.barrier()
    finally:
        td.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_count_every_token():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    for r in res:
        assert abs(r[2] - 2 * 100 / 0.015) < 1e-6


def test_single_process_is_the_identity():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_throughput(1, 200, 400.0) == 500.0


def test_reference_arm_runs_on_rank_zero_only():
    # ranks other than 0 return before building the oracle model (they exit 0 without work)
    args = SimpleNamespace(warmup=3, steps=1, gpus=2)
    assert bench.run_reference(args, cfg=None, rank=1, world=2) is None
