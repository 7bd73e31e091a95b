"""Multi-rank host logic on CPU: LPT user sharding and output reassembly,
with world-size-2 gloo process groups.  Each rank computes its share with the
fp64 oracle (the stand-in for its GPU); the gathered result must equal the
single-process oracle on the whole batch, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from latent_attention_jagged_b200 import cost
from latent_attention_jagged_b200.sharding import (gather_outputs, lpt_partition, make_shard,
                                                   shard_batch, user_flops)
from workloads import Dims, Workload, make_inputs, workload


def test_user_flops_sum_to_batch_total():
    inp = make_inputs(workload("skewed"), batch=64)
    tot = user_flops(inp.lengths, inp.dims).sum()
    assert abs(tot - cost.total_flops(inp.lengths, inp.dims)) <= 1e-6 * tot


def test_lpt_partition_covers_and_balances():
    rng = np.random.default_rng(0)
    costs = rng.lognormal(5.5, 0.8, size=513)
    for world in (1, 2, 3, 8):
        parts = lpt_partition(costs, world)
        allu = np.sort(np.concatenate(parts))
        assert np.array_equal(allu, np.arange(costs.size))
        loads = np.array([costs[p].sum() for p in parts])
        # LPT bound: max load <= mean load + largest item
        assert loads.max() <= costs.sum() / world + costs.max() + 1e-9


def test_make_shard_rows_and_offsets():
    offsets = np.array([0, 3, 3, 7, 8], dtype=np.int64)
    sh = make_shard(offsets, np.array([0, 2, 3]))
    assert sh.offsets.tolist() == [0, 3, 7, 8]
    assert sh.rows.tolist() == [0, 1, 2, 3, 4, 5, 6, 7]
    sh = make_shard(offsets, np.array([1, 3]))
    assert sh.offsets.tolist() == [0, 0, 1]
    assert sh.rows.tolist() == [7]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, results):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dims = Dims(d=16, heads=2, d_head=8, rank=12, d_ctx=5, n_q=3, keep=(9, 4), dtype="fp32")
        wl = Workload(name="t", dims=dims, batch=11, lengths=("uniform", 0, 20), seed=5)
        inp = make_inputs(wl)
        shards = shard_batch(inp.offsets, dims, world)
        sh = shards[rank]
        local = oracle.forward(inp, users=sh.users.tolist()) if sh.users.size else \
            np.zeros((0, dims.n_q, dims.d))
        full = gather_outputs(torch.as_tensor(local), sh, inp.batch)
        if rank == 0:
            ref = oracle.forward(inp)
            results.put(bool(np.array_equal(full.numpy(), ref)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_gloo_shard_and_gather_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=100)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5) is True
