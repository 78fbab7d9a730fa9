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


def test_reference_arm_times_exactly_k_steps_after_w(monkeypatch, capsys):
    """`bench.py --impl reference` runs the oracle W untimed steps, then
    exactly K timed steps, and prints one JSON line on the metric's unit
    with the reference-arm keys (on a small workload, on the CPU)."""
    import json
    import types
    b = _bench()
    from oracle import oracle as O
    calls = []
    real = O.layer

    def counting(*a, **k):
        calls.append(1)
        return real(*a, **k)

    monkeypatch.setattr(O, "layer", counting)
    monkeypatch.setenv("RANK", "0")
    args = types.SimpleNamespace(config="tiny-fp32-r1", steps=4, warmup=2, gpus=1)
    b.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert len(calls) == 1 + 2 + 4   # first touch, W warm-up, K timed
    assert line["impl"] == "reference" and line["steps"] == 4 and line["warmup"] == 2
    assert line["unit"] == b.UNIT and line["higher_is_better"] is False and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and "2 warm-up and 4 timed steps" in line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": b.UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
