"""bench.py's multi-rank plumbing on CPU: two gloo ranks, each timing a
different (fake) step, must agree on the max-over-ranks time and on the
whole-job rate computed from it.  The path itself has no exchange step, so
the barrier and this max are the only collectives a replica run makes."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, backend="gloo")
    try:
        d.barrier()
        ms = d.max(10.0 + 5.0 * rank)  # rank r's step took 10 + 5r ms
        rate = bench.whole_job_rate(131072, d.world, ms)
        d.barrier()
        q.put((rank, d.world, ms, rate))
    finally:
        d.close()


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, w, ms, rate in got:
        assert w == world
        assert ms == 15.0                       # the slowest rank's time
        assert rate == 2 * 131072 / 0.015       # all ranks' tokens / that time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    d = bench.Dist(1)
    assert d.pg is None and d.world == 1
    assert d.max(3.5) == 3.5
    d.barrier()
    d.close()
    assert bench.whole_job_rate(16, 1, 0.25) == 64000.0
