"""The multi-GPU path of bench.py is replicas: every rank runs its own layer
and the job's time is the maximum over ranks.  Its host logic runs here on
CPU with two gloo ranks (no GPU): rank discovery from the launcher's
environment, per-rank seeds, and the max-over-ranks reduction that every rank
must reach in the same order."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        # each replica draws its own routing (seed = rank)
        ids = synth.make_moe_inputs(synth.CONFIGS["tiny"], seed=r, weights=False)["topk_ids"]
        gathered = [torch.zeros_like(ids) for _ in range(world)]
        dist.all_gather(gathered, ids)
        distinct = not torch.equal(gathered[0], gathered[1])
        # per-rank times: the job time is the slowest rank's
        mine = [10.0 + rank, 5.0 - rank]
        got = bench.max_over_ranks(mine, dist)
        dist.barrier()
        results[rank] = (got, distinct)
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        got, distinct = results[r]
        assert got == [11.0, 5.0]
        assert distinct


def test_max_over_ranks_without_group():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
