"""The N > 1 host logic of bench.py on CPU: two gloo ranks (replicas) agree
on the slowest rank's time and on the whole-job throughput, and a rank that
never joins ends the others' collective with an error instead of a hang."""
import datetime
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    import bench
    m = bench.max_over_ranks(local_ms[rank], world)
    v = bench.whole_job_tflops(world, 1.0e12, 10, m)
    out.put((rank, m, v))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_agree_on_the_slowest_time_and_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    local_ms = [120.0, 150.0]
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=5) for _ in range(world))
    for rank, m, v in got:
        assert m == 150.0
        # 2 ranks x 10 steps x 1 TFLOP in 0.15 s
        assert abs(v - 2 * 10 * 1.0 / 0.150) < 1e-9


def _lonely_rank(port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        dist.init_process_group("gloo", rank=0, world_size=2, timeout=datetime.timedelta(seconds=3))
        t = torch.zeros(1)
        dist.all_reduce(t)
        out.put("returned")
    except Exception as e:  # the peer never joins: a bounded wait ends in an error
        out.put(type(e).__name__)


def test_a_missing_rank_ends_in_an_error_not_a_hang():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    p = ctx.Process(target=_lonely_rank, args=(port, out))
    p.start()
    p.join(timeout=120)
    if p.is_alive():
        p.kill()
        pytest.fail("the lone rank did not give up")
    assert out.get(timeout=5) != "returned"
