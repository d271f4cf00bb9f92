"""The multi-rank host path of bench.py on CPU: two spawned ranks rendezvous over gloo (the
backend bench.py picks without CUDA), agree on the slowest rank's time through
max_over_ranks, and pass the barriers that bracket the timed region.  The replicas exchange
nothing else: the sequences of different ranks are independent."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, w, _ = bench.dist_setup(world)
    bench.barrier(w)
    slowest = bench.max_over_ranks(times[rank], w, "cpu")
    bench.barrier(w)
    out.put((r, w, dist.get_backend(), slowest))
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    times = [12.5, 31.25]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 and g[2] == "gloo" for g in got)
    assert all(g[3] == max(times) for g in got)
    assert all(p.exitcode == 0 for p in procs)
