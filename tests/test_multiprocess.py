"""The N > 1 plumbing of bench.py on CPU: two gloo ranks, each timing its own
replica row, reduce to the slowest rank's times (the step time of the job), and
draw different replica inputs.  The solver's data path has no collective."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as W
        mine = [1.0 + rank, 10.0 - rank, 0.5 * rank]
        got = bench.max_over_ranks(dist, mine)
        w = W.Workload("tiny", 1, 1000, 10.0, 0.1, "normal", "")
        r = W.scores(w, seed=rank)[0]
        out.put((rank, got, float(r[:4].sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, got0, s0), (r1, got1, s1) = res
    assert got0 == got1 == [2.0, 10.0, 0.5]
    assert s0 != s1            # each rank solves a different replica row


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(None, [3.0, 4.0]) == [3.0, 4.0]
