"""Multi-process path of bench.py on CPU: two gloo ranks stand in for two
GPUs.  The decode path does not shard (each GPU runs a whole replica of the
model on its own batch), so the only cross-rank step is the timing reduction:
every rank's device time goes through an element-wise maximum, and the
whole-job rate counts the units of all ranks over the slowest rank's time."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        bench = _bench()
        # rank-specific timings (ms): total, prefill, decode, e2e, wall
        mine = torch.tensor([100.0 + rank, 10.0 * (2 - rank), 50.0 + 3 * rank, 7.0, 1.5 * (rank + 1)],
                            dtype=torch.float64)
        got = bench.max_over_ranks(mine.clone(), world).tolist()
        rate = bench.whole_job_rate(1024, world, got[2])
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, got, rate))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e), None))


def test_timing_reduction_takes_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [101.0, 20.0, 53.0, 7.0, 3.0]
    for rank, got, rate in results:
        assert not isinstance(got, str), got
        assert got == want, (rank, got)
        # 2 ranks x 1024 tokens over the slowest decode time (53 ms)
        assert rate == pytest.approx(2 * 1024 / 0.053)


def test_single_rank_needs_no_process_group():
    bench = _bench()
    v = torch.tensor([3.0, 1.0], dtype=torch.float64)
    assert bench.max_over_ranks(v, 1).tolist() == [3.0, 1.0]
    assert bench.whole_job_rate(10, 1, 1000.0) == pytest.approx(10.0)
