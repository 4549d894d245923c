"""The benchmark's multi-process plumbing on CPU: two ranks over gloo, as
torchrun launches them (one process per GPU on a real node).  Each rank runs
an independent replica of the workload; the only collectives are the barrier
around the timed region and the max over ranks of the elapsed time."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("mglu_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    bench = _bench_module()
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    elapsed = 10.0 * (rank + 1)         # per-rank timed region, ms
    worst = d.max(elapsed)              # every rank must agree on the slowest
    T, K = 4, 50
    value = d.world * T * K / (worst / 1000.0)
    d.barrier()
    d.close()
    q.put((rank, d.world, worst, value))


@pytest.mark.parametrize("world", [2])
def test_two_ranks_agree_on_max_and_aggregate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(world))
    for _, w, worst, value in res:
        assert w == world
        assert worst == 10.0 * world        # the slowest rank's time
        assert value == pytest.approx(world * 4 * 50 / (worst / 1000.0))


def test_single_process_needs_no_group():
    bench = _bench_module()
    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist()
    d.init("gloo")
    assert d.world == 1 and not d.pg
    d.barrier()
    assert d.max(3.5) == 3.5
    d.close()
