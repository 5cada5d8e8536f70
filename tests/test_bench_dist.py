"""The benchmark's multi-process plumbing on CPU: two gloo ranks take the barrier
and the max-over-ranks of their timings, as bench.py does under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, l = bench.dist_env()
    assert (w, r, l) == (world, rank, rank)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    m = bench.max_over_ranks(10.0 + rank, world)
    out[rank] = m
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_and_max():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _rank_reduce(rank, world, port, out):
    """Each rank makes its own dW per linear (seeded by rank), the reducer sums them over
    the ranks and leaves rank r the rows [r*out/N, (r+1)*out/N)."""
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    shapes = [(256, 128), (512, 384)]
    red = bench.DpGradReducer(shapes, world, "cpu")

    def grad(r, i, dout, din):
        g = torch.Generator().manual_seed(1000 * r + i)
        # values on a coarse grid so that BF16 sums of two ranks are exact
        return (torch.randint(-64, 64, (dout, din), generator=g).float() / 16).to(torch.bfloat16)

    for i, (dout, din) in enumerate(shapes):
        red.launch(i, grad(rank, i, dout, din))
    red.wait()
    ok = True
    for i, (dout, din) in enumerate(shapes):
        lo, hi = bench.DpGradReducer.rows(dout, world, rank)
        want = sum(grad(r, i, dout, din).float() for r in range(world))[lo:hi]
        ok = ok and torch.equal(red.shards[i].float(), want)
    out[rank] = ok
    dist.destroy_process_group()


def test_two_gloo_ranks_dw_reduce_scatter():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_reduce, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {0: True, 1: True}
