"""Multi-process (gloo, world size 2, CPU) checks of the data-parallel replica bookkeeping:
per-rank batches differ, the timing is the maximum over ranks, and the throughput counts all
ranks' tokens.  No collective touches the data path of the layer itself."""

import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mxfp4_quantized_moe_b200 import inputs, replicas


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank draws its own token batch; the weights come from the shared seed
        base = inputs.make_layer(8, 64, 64, 4, 2, 7)
        mine = inputs.make_layer(8, 64, 64, 4, 2, replicas.batch_seed(7, rank))
        # a stand-in step time that differs per rank
        ms = 10.0 + 5.0 * rank
        m = replicas.max_over_ranks(ms)
        value = replicas.aggregate_tokens_per_s(8, 3, m, world)
        xs = [torch.zeros_like(mine["x"].float()) for _ in range(world)]
        dist.all_gather(xs, mine["x"].float())
        q.put((rank, m, value, torch.equal(base["gu_blocks"], mine["gu_blocks"]),
               bool(torch.equal(xs[0], xs[1]))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_aggregate():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, value, _, same_x in res:
        assert m == pytest.approx(15.0)  # max over ranks, on every rank
        assert value == pytest.approx(8 * world * 3 / 0.015)
        assert not same_x  # the two ranks drew different token batches
    # rank 0 keeps the base seed; the weight draw does not depend on the rank offset for rank 0
    assert res[0][3]


def test_single_process_is_identity():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.batch_seed(5, 0) == 5
    assert replicas.aggregate_tokens_per_s(100, 2, 1000.0, 1) == pytest.approx(200.0)
