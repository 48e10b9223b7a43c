"""The multi-rank paths, on CPU with the gloo backend.

`bench.py --gpus N` runs one independent replica per rank (weak scaling: the
hot path has no cross-rank exchange) and reports the slowest rank's time and
the sum of all ranks' work; the first test checks its barrier and
max-over-ranks reduction.  The context-split decode (one cache's rows shared
among ranks) does exchange: every rank gathers all (out, lse) pairs and
merges them; the second test runs that exchange on two gloo ranks, with the
oracle computing each rank's part on the host.  The context-split probe (one
context's keys shared among ranks) exchanges twice: the probe rows' partial
(max, Z), then every rank's top-k candidates; the third test runs both
gathers on two gloo ranks against the oracle's whole-context index list.
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


def _cp_worker(rank, world, port, q):
    """One rank of a context-split decode: decode this rank's rows of the
    shared cache (the oracle stands in for the GPU decode on the host), gather
    every rank's (out, lse) and merge."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from kv_cache_vertical_b200 import hq
        from kv_cache_vertical_b200.synth import F5, Workload, make_inputs
        from test_context_split import _sub, merge_np
        w = Workload("cp", "decode", 1, 8, 2, 128, 2500, 128, F5, 4, 123)
        x = make_inputs(w)                       # the same seed on every rank: one cache
        c = oracle.pack_kv(x["k"], x["v"], x["planted"].numpy(), w.window, 4)
        part = hq.context_split_plan(c["n_lo"], c["n_hi"], world)[rank]
        out, lse = oracle.decode_attn(x["q"], _sub(c, *part), w.Hkv)
        outs = [torch.empty(out.shape, dtype=torch.float64) for _ in range(world)]
        lses = [torch.empty(lse.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(outs, torch.from_numpy(out))
        dist.all_gather(lses, torch.from_numpy(lse))
        merged, mlse = merge_np([t.numpy() for t in outs], [t.numpy() for t in lses])
        full, full_lse = oracle.decode_attn(x["q"], c, w.Hkv)
        q.put((rank, float(np.abs(merged - full).max()), float(np.abs(mlse - full_lse).max()),
               part[1] - part[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_context_split_decode():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[3] > 0 for r in results)              # both ranks hold low rows
    for rank, err, lse_err, _ in results:
        assert err < 1e-12 and lse_err < 1e-12, (rank, err, lse_err)


def _probe_cp_worker(rank, world, port, q):
    """One rank of a context-split probe: this rank's keys only (a restatement
    of the probe definition stands in for the GPU passes on the host); the
    probe rows' (max, Z) are gathered and merged, then every rank's top-k
    candidates are gathered and merged."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from kv_cache_vertical_b200 import hq
        from kv_cache_vertical_b200.synth import F5, Workload, make_inputs
        from test_context_split import (merge_candidates_np, merge_stats_np, probe_shard_np,
                                        shard_candidates_np)
        w = Workload("pcp2", "decode", 1, 8, 2, 64, 900, 64, F5, 4, 321)
        x = make_inputs(w)                       # the same seed on every rank: one context
        off, n = hq.probe_context_plan(w.L, world)[rank]
        ks = x["k"][:, :, off:off + n]
        m, z = probe_shard_np(x["q_probe"], ks, off, w.L, w.Hkv)
        ms = [torch.empty(m.shape, dtype=torch.float64) for _ in range(world)]
        zs = [torch.empty(z.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(ms, torch.from_numpy(m))
        dist.all_gather(zs, torch.from_numpy(z))
        stats = merge_stats_np([(a.numpy(), b.numpy()) for a, b in zip(ms, zs)])
        score = probe_shard_np(x["q_probe"], ks, off, w.L, w.Hkv, stats)
        ci, cs = shard_candidates_np(score, off, w.L, w.window, w.k_vert)
        cis = [torch.empty(ci.shape, dtype=torch.int64) for _ in range(world)]
        css = [torch.empty(cs.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(cis, torch.from_numpy(ci))
        dist.all_gather(css, torch.from_numpy(cs))
        idx = merge_candidates_np([t.numpy() for t in cis], [t.numpy() for t in css], w.L,
                                  w.window, w.k_vert)
        ref = oracle.topk(oracle.probe_scores(x["q_probe"], x["k"], w.Hkv), w.window, w.k_vert)
        q.put((rank, bool(np.array_equal(idx, ref)), n))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_context_split_probe():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_probe_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same, n in results:
        assert n > 0 and same, (rank, same, n)
