"""The multi-rank part of the benchmark on CPU: two gloo ranks, the way
`bench.py --gpus 2` aggregates independent replicas (no data-path
collective): every rank's timed totals reduced to the max over ranks, and
the whole job's value counting the layer-steps of all ranks."""

import importlib.util
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    b = _bench()
    # each rank's own totals: rank 1 is the slower replica in the first, rank 0 in the second
    mine = (100.0 + 25.0 * rank, 80.0 - 10.0 * rank)
    got = b.job_times(mine[0], mine[1], world, "cpu")
    out.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_max_and_count_every_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the same totals: the slowest rank's of each
    assert res[0] == res[1] == (125.0, 80.0)
    b = _bench()
    # 1000 steps of 1 layer on each of 2 ranks in 125 ms: 62.5 us per layer-step of the job
    assert b.job_value(res[0][0], 1000, 1, 2) == pytest.approx(62.5)
    # one rank: no collective, the value is its own time per layer-step
    assert b.job_times(3.0, 4.0, 1, "cpu") == (3.0, 4.0)
    assert b.job_value(400.0, 100, 4, 1) == pytest.approx(1000.0)
