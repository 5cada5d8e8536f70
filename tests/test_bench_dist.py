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


def _rank_reduce_fp32(rank, world, port, out):
    """Each rank holds its own token shard of X and dY and computes the oracle's wgrad
    over that shard as its local FP32 main gradient; the package's DpGradReducer sums
    the FP32 gradients over the ranks (gloo reduce-scatter).  Rank r's rows must equal
    the oracle's wgrad over the concatenated tokens within the FP32 rounding of the
    exchange: each local gradient rounded once to binary32 plus one binary32 addition,
    at most 3 * 2^-24 * sum_k |ahat_k bhat_k| per output."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from blockwise_fp8_linear_b200 import synth
    from blockwise_fp8_linear_b200.dp import DpGradReducer

    T, din, dout = 512, 256, 384                    # 256 tokens per rank: two 128-groups
    X = synth.normal_bf16(T, din, 1.0, seed=synth.seed_for(77, 0), outliers=True)
    dY = synth.normal_bf16(T, dout, 1e-3, seed=synth.seed_for(77, 2))

    def wgrad(x, dy):
        a, sa = oracle.quant_act_t(np.ascontiguousarray(dy))
        b, sb = oracle.quant_act_t(np.ascontiguousarray(x))
        return oracle.gemm(oracle.WGRAD, a, sa, b, sb, dout, din, x.shape[0])

    lo, hi = rank * T // world, (rank + 1) * T // world
    local, _ = wgrad(X[lo:hi], dY[lo:hi])
    red = DpGradReducer([(dout, din)], world, "cpu")
    red.launch(0, torch.from_numpy(local.astype(np.float32)))
    red.wait()
    full, asum = wgrad(X, dY)
    r0, r1 = DpGradReducer.rows(dout, world, rank)
    got = red.shards[0].double().numpy()
    err = np.abs(got - full[r0:r1])
    out[rank] = bool(np.all(err <= 3 * 2.0 ** -24 * asum[r0:r1])) and bool(np.any(got != 0))
    dist.destroy_process_group()


def test_two_gloo_ranks_fp32_main_grad_reduce_scatter():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_reduce_fp32, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert dict(out) == {0: True, 1: True}


def test_reducer_rejects_bad_shapes():
    import torch
    from blockwise_fp8_linear_b200.dp import DpGradReducer
    import pytest
    with pytest.raises(ValueError):
        DpGradReducer([(130, 128)], 4, "cpu")
    red = DpGradReducer([(256, 128)], 2, "cpu")
    with pytest.raises(ValueError):
        red.launch(0, torch.zeros(256, 128, dtype=torch.bfloat16))   # not the FP32 main grad
    with pytest.raises(ValueError):
        red.launch(0, torch.zeros(128, 256))
