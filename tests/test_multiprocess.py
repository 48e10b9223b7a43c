"""The multi-rank plumbing of bench.py, on CPU with the gloo backend.

`bench.py --gpus N` runs one independent replica per rank (weak scaling: the
hot path has no cross-rank exchange) and reports the slowest rank's time and
the sum of all ranks' work.  These tests run two gloo ranks on the host and
check the barrier and the max-over-ranks reduction that the GPU run uses.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        # each rank reports its own time; the job time is the slowest rank's
        t = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        # every rank runs a replica with its own seed: distinct inputs per rank
        w = bench.WL.replace(seed=bench.WL.seed + rank, L=256, Hq=4, Hkv=2)
        from kv_cache_vertical_b200.synth import make_inputs
        x = make_inputs(w)
        digest = float(x["k"].float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        q.put((rank, t, digests))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_time_and_distinct_replicas():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, digests in results:
        assert t == 10.0 + (world - 1)          # max over ranks, seen by every rank
        assert digests[0] != digests[1]         # replicas draw different inputs
