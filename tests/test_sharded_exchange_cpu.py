"""The exchange steps of the context-sharded decode on two CPU ranks over gloo.

Each rank stands for one shard.  exchange_candidates and exchange_partials must give every
rank the same stacks, in rank order (the merge is then identical on every rank, and shard r's
candidates sit at position r).  The tensors carry rank-dependent values, including -1 padding
and an empty shard (count 0, m = -inf), as the kernels write them; nothing here runs a
kernel."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B_, K_ = 3, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local(rank):
    import torch
    g = torch.Generator().manual_seed(100 + rank)
    cs = torch.rand((B_, K_), generator=g)
    ci = (torch.arange(B_ * K_, dtype=torch.int32).view(B_, K_) + 1000 * rank)
    cc = torch.tensor([K_, 5 - rank, 0], dtype=torch.int32)
    ci[1, cc[1]:] = -1
    ci[2, :] = -1
    po = torch.randn((B_, 24, 128), generator=g)
    pm = torch.randn((B_, 24), generator=g)
    pm[2] = float("-inf") if rank == 1 else pm[2]
    pl = torch.rand((B_, 24), generator=g)
    return cs, ci, cc, po, pm, pl


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from block_sparse_attention_40_b200 import sharded as S
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    cs, ci, cc, po, pm, pl = _local(rank)
    gcs, gci, gcc = S.exchange_candidates(cs, ci, cc)
    gpo, gpm, gpl = S.exchange_partials(po, pm, pl)
    ok = True
    for r in range(world):
        want = _local(r)
        for got, w in zip((gcs[r], gci[r], gcc[r], gpo[r], gpm[r], gpl[r]), want):
            ok = ok and got.dtype == w.dtype and torch.equal(got, w)
    shapes = [tuple(t.shape) for t in (gcs, gci, gcc, gpo, gpm, gpl)]
    out.put((rank, ok, shapes))
    dist.destroy_process_group()


def test_two_ranks_gather_candidates_and_partials_in_rank_order():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
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
    assert all(g[1] for g in got)
    assert got[0][2] == [(2, B_, K_), (2, B_, K_), (2, B_), (2, B_, 24, 128), (2, B_, 24),
                         (2, B_, 24)]
    assert all(p.exitcode == 0 for p in procs)
