"""Whole-matrix sharding (host plumbing): the ownership plan, the flat weight
layout and the all-gather exchange, on CPU.  The multi-rank cases run two
gloo ranks as processes; each rank stands in for its GPU step with the fp64
oracle on the matrices it owns, then the slices are exchanged, and every rank
must end with the weights a single process gets by stepping all matrices."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as orc
import workloads
from dimuon_optimizer_b200 import sharded

MIXED = (workloads.gpt2_small_shapes(layers=2) + workloads.lora_shapes(8, projections=6) +
         [(4096, 4096), (1000, 3), (7, 5000)])


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_plan_complete_aligned_disjoint(world):
    plan = sharded.plan_shards(MIXED, world)
    assert len(plan.owner) == len(MIXED) and set(plan.owner) <= set(range(world))
    spans = []
    for i, (r, c) in enumerate(MIXED):
        o = plan.offset[i]
        assert o % sharded.ALIGN_ELEMS == 0
        k = plan.owner[i]
        # inside the owner's slice
        assert k * plan.slice_elems <= o and o + r * c <= (k + 1) * plan.slice_elems
        spans.append((o, o + r * c))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))  # no overlap
    assert sorted(i for k in range(world) for i in plan.owned(k)) == list(range(len(MIXED)))


@pytest.mark.parametrize("world", [2, 4, 8])
def test_plan_balanced(world):
    """Greedy longest-first: no rank carries more than the mean plus the
    largest single matrix."""
    plan = sharded.plan_shards(MIXED, world)
    loads = [plan.load(k) for k in range(world)]
    biggest = max(sharded.matrix_cost(r, c) for r, c in MIXED)
    assert max(loads) <= sum(loads) / world + biggest + 1e-15


def test_plan_deterministic():
    a = sharded.plan_shards(MIXED, 4)
    b = sharded.plan_shards(list(MIXED), 4)
    assert a == b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPES = [(24, 40), (40, 24), (8, 96), (96, 4), (33, 33), (5, 70)]


def _inputs():
    rng = np.random.default_rng(123)
    W = [0.02 * rng.standard_normal(s) for s in SHAPES]
    G = [rng.standard_normal(s) for s in SHAPES]
    M = [rng.standard_normal(s) for s in SHAPES]
    return W, G, M


def _stepped_all():
    W, G, M = _inputs()
    h = orc.HParams(mu=0.9, lr=0.05, weight_decay=0.01)
    return [orc.muon_step(W[i], G[i], M[i], h).W for i in range(len(SHAPES))]


def _rank_main(rank, world, port, errq):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        plan = sharded.plan_shards(SHAPES, world)
        sw = sharded.ShardedWeights(plan, dtype=torch.float64, device="cpu")
        W, G, M = _inputs()
        for i in range(len(SHAPES)):
            sw.views[i].copy_(torch.from_numpy(W[i]))
        h = orc.HParams(mu=0.9, lr=0.05, weight_decay=0.01)
        for i in plan.owned(rank):  # this rank's "GPU step"
            sw.views[i].copy_(torch.from_numpy(orc.muon_step(W[i], G[i], M[i], h).W))
        # matrices owned elsewhere are stale here until the exchange
        sw.gather(rank)
        want = _stepped_all()
        for i in range(len(SHAPES)):
            np.testing.assert_array_equal(sw.views[i].numpy(), want[i])
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_exchange_gloo(world):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    errors = []
    while not errq.empty():
        errors.append(errq.get())
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def test_single_rank_gather_is_noop():
    plan = sharded.plan_shards(SHAPES, 1)
    sw = sharded.ShardedWeights(plan, dtype=torch.float32, device="cpu")
    sw.views[0].fill_(3.0)
    sw.gather(0)
    assert float(sw.views[0][0, 0]) == 3.0


def _rank_main_dp(rank, world, port, errq):
    """Data-parallel flavour: every rank holds its own local gradients in the
    flat layout; one reduce-scatter gives each owner the mean over ranks, the
    owner steps (the oracle stands in for the GPU step), the weights are
    all-gathered, and every rank must end with the single-process step on
    the mean gradient."""
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        plan = sharded.plan_shards(SHAPES, world)
        sw = sharded.ShardedWeights(plan, dtype=torch.float64, device="cpu")
        sg = sharded.ShardedGrads(plan, dtype=torch.float64, device="cpu")
        W, _, M = _inputs()
        local = _local_grads(world)
        for i in range(len(SHAPES)):
            sw.views[i].copy_(torch.from_numpy(W[i]))
            sg.views[i].copy_(torch.from_numpy(local[rank][i]))
        sg.reduce(rank)
        h = orc.HParams(mu=0.9, lr=0.05, weight_decay=0.01)
        mean = [sum(local[q][i] for q in range(world)) / world for i in range(len(SHAPES))]
        for i in plan.owned(rank):
            np.testing.assert_allclose(sg.views[i].numpy(), mean[i], rtol=1e-13, atol=1e-14)
            sw.views[i].copy_(torch.from_numpy(
                orc.muon_step(W[i], sg.views[i].numpy(), M[i], h).W))
        sw.gather(rank)
        for i in range(len(SHAPES)):
            want = orc.muon_step(W[i], mean[i], M[i], h).W
            np.testing.assert_allclose(sw.views[i].numpy(), want, rtol=1e-10, atol=1e-12)
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


def _local_grads(world):
    rng = np.random.default_rng(321)
    return [[rng.standard_normal(s) for s in SHAPES] for _ in range(world)]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_grad_reduce_scatter_gloo(world):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_dp, args=(r, world, port, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    errors = []
    while not errq.empty():
        errors.append(errq.get())
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def test_grads_layout_matches_weights():
    plan = sharded.plan_shards(SHAPES, 3)
    sw = sharded.ShardedWeights(plan, dtype=torch.float32, device="cpu")
    sg = sharded.ShardedGrads(plan, dtype=torch.float32, device="cpu")
    assert sg.flat.numel() == sw.flat.numel()
    for a, b in zip(sg.views, sw.views):
        assert a.shape == b.shape
        assert a.storage_offset() == b.storage_offset()
    # one rank: nothing to reduce, no process group needed
    one = sharded.ShardedGrads(sharded.plan_shards(SHAPES, 1), dtype=torch.float32, device="cpu")
    one.views[0].fill_(2.0)
    one.reduce(0)
    assert float(one.views[0][0, 0]) == 2.0
