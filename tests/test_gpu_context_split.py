"""GPU parity of the context-split paths, their ranks run one after another on
one GPU.  Decode: each part of the plan is decoded through a row view of one
packed cache, the parts are merged by hq_decode_merge, and the result is
compared with the oracle's decode of the whole cache (the CUDA path's cache is
the oracle's, bit for bit, as the pack tests show).  Probe: each rank's keys
go through the shard entry points, the merges pick the context's columns, and
the index lists are compared with the oracle's whole-context probe."""
import numpy as np
import pytest
import torch

import oracle
from hq_testutil import assert_close, to_dev
from kv_cache_vertical_b200.synth import F5, WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


def run_split(w: Workload, R: int, fmt=0):
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    idx = x["planted"].numpy()
    cache = H.pack_kv(d["k"], d["v"], torch.from_numpy(idx).cuda(), w.window, w.bits, fmt=fmt)
    ref = oracle.pack_kv(x["k"], x["v"], idx, w.window, w.bits, 32, fmt)
    full, full_lse = oracle.decode_attn(x["q"], ref, w.Hkv)
    outs, lses = [], []
    for rows in H.context_split_plan(cache.n_lo, cache.n_hi, R):
        part = cache.rows_part(*rows)
        if part.n_lo + part.n_hi == 0:
            outs.append(torch.zeros(w.B, w.Hq, w.D, device="cuda"))
            lses.append(torch.full((w.B, w.Hq), float("-inf"), device="cuda"))
            continue
        o, l = H.decode_attn(d["q"], part, w.Hkv, want_lse=True)
        outs.append(o)
        lses.append(l)
    out, lse = H.decode_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), full, f"context split R={R}")
    assert np.allclose(lse.cpu().numpy(), full_lse, atol=1e-4, rtol=1e-5)


@pytest.mark.parametrize("R", [2, 3, 4])
@pytest.mark.parametrize("bits,D", [(4, 128), (8, 128), (4, 64)])
def test_context_split_matches_whole_cache(R, bits, D):
    w = Workload("cs", "decode", 2, 8, 2, D, 6001, 128, F5, bits, 11 * R + bits + D)
    run_split(w, R)


def test_context_split_fp8_few_low_rows():
    # 3 ranks over a cache with few low rows: some ranks read bf16 rows only
    w = Workload("cs_fp8", "decode", 1, 4, 1, 128, 400, 256, F5, 8, 3)
    H = hq()
    assert any(lo1 == lo0 for lo0, lo1, _, _ in
               H.context_split_plan(400 - 256 - w.k_vert, 256 + w.k_vert, 3))
    run_split(w, 3, fmt=1)


def test_context_split_more_ranks_than_pairs_rows():
    # 8 ranks over a short cache: several parts are small, one may be empty
    w = Workload("cs_short", "decode", 1, 8, 2, 128, 700, 128, F5, 4, 8)
    run_split(w, 8)


def test_context_split_llama8b_full_size():
    run_split(WORKLOADS["llama8b_decode_32k"], 2)


def test_merge_kernel_against_numpy():
    H = hq()
    g = torch.Generator().manual_seed(5)
    R, B, Hq, D = 5, 3, 8, 128
    po = torch.randn(R, B, Hq, D, generator=g)
    pl = torch.randn(R, B, Hq, generator=g) * 4
    pl[1, 0, :] = float("-inf")                       # an empty part
    pl[:, 2, 3] = float("-inf")                       # every part empty for one head
    out, lse = H.decode_merge(po.cuda(), pl.cuda())
    torch.cuda.synchronize()
    m = pl.double().amax(0)
    wgt = torch.exp(pl.double() - torch.where(torch.isinf(m), torch.zeros_like(m), m))
    ref = (wgt[..., None] * po.double()).sum(0) / wgt.sum(0)[..., None]
    ref[2, 3] = 0.0
    got = out.cpu().double()
    assert torch.allclose(got, ref, atol=1e-5, rtol=1e-5)
    assert torch.isinf(lse[2, 3].cpu()) and lse[2, 3].item() < 0
    ok = torch.ones(B, Hq, dtype=torch.bool)
    ok[2, 3] = False
    ref_lse = m + torch.log(wgt.sum(0))
    assert torch.allclose(lse.cpu().double()[ok], ref_lse[ok], atol=1e-5)


# ---------------------------------------------------------------------------
# Context-split probe: each rank's keys through the shard entry points, the
# ranks one after another on one GPU, merged by the merge entry points;
# compared with the oracle's probe of the whole context (index sets equal
# modulo ties) and with the single-GPU probe.
# ---------------------------------------------------------------------------

def run_probe_split(w: Workload, R: int):
    from hq_testutil import assert_index_sets
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    qp, k = d["q_probe"], d["k"]
    plan = H.probe_context_plan(w.L, R)
    parts = [H.probe_shard_stats(qp, k[:, :, o:o + n].contiguous(), o, w.L) for o, n in plan]
    stats = H.probe_merge_stats(torch.stack(parts))
    cand = [H.probe_shard_topk(qp, k[:, :, o:o + n].contiguous(), o, w.L, w.window, w.k_vert, stats)
            for o, n in plan]
    idx = H.probe_merge_topk(torch.stack([c[0] for c in cand]), torch.stack([c[1] for c in cand]),
                             w.L, w.window)
    one = H.probe_vertical(qp, k, w.window, w.k_vert)
    torch.cuda.synchronize()
    sc = oracle.probe_scores(x["q_probe"], x["k"], w.Hkv)
    ref = oracle.topk(sc, w.window, w.k_vert)
    assert_index_sets(idx.cpu().numpy(), ref, sc, w.window)
    assert_index_sets(one.cpu().numpy(), ref, sc, w.window)
    # every rank's candidates are context positions before the window, or -1
    for (o, n), (ci, _) in zip(plan, cand):
        c = ci.cpu().numpy()
        v = c[c >= 0]
        assert ((v >= o) & (v < min(o + n, w.L - w.window))).all()


@pytest.mark.parametrize("R", [1, 2, 3])
@pytest.mark.parametrize("D", [64, 128])
def test_probe_split_matches_whole_context(R, D):
    w = Workload("pcp", "decode", 2, 8, 2, D, 5003, 128, F5, 4, 600 + R + D)
    run_probe_split(w, R)


def test_probe_split_rank_without_candidates():
    # 4 ranks over 300 keys (75 each) with a 100-key window: the last rank's
    # keys all lie in the window, so it has no candidates, only row stats
    w = Workload("pcp_w", "decode", 1, 4, 1, 128, 300, 100, F5, 4, 77)
    run_probe_split(w, 4)


def test_probe_split_llama8b_32k():
    w = WORKLOADS["llama8b_decode_32k"]
    run_probe_split(w, 4)


# ---------------------------------------------------------------------------
# Sharded context split: every rank packs and holds only its part of the
# cache's rows (hq_pack_kv_part), appends go to the rank holding the window
# (hq_kv_append_part), and the two exchange functions run end to end with one
# process per rank.
# ---------------------------------------------------------------------------

from hq_testutil import assert_index_sets, assert_pack_equal, cache_to_np  # noqa: E402


def _rows(c: dict, lo0, lo1, hi0, hi1) -> dict:
    out = {n: c[n][:, :, lo0:lo1] for n in ("k_codes", "v_codes", "k_sz", "v_sz")}
    out.update(k_hi=c["k_hi"][:, :, hi0:hi1], v_hi=c["v_hi"][:, :, hi0:hi1],
               lo_pos=c["lo_pos"][:, :, lo0:lo1] if c["lo_pos"] is not None else None)
    return out


@pytest.mark.parametrize("R", [2, 3])
@pytest.mark.parametrize("bits,D,fmt", [(4, 128, 0), (8, 64, 0), (8, 128, 1)])
def test_pack_parts_are_the_whole_cache_rows(R, bits, D, fmt):
    H = hq()
    w = Workload("pp", "decode", 2, 8, 2, D, 5003, 128, F5, bits, 700 + R + D + fmt)
    d = to_dev(make_inputs(w))
    idx = d["planted"]
    whole = H.pack_kv(d["k"], d["v"], idx, w.window, bits, fmt=fmt)
    wc = cache_to_np(whole)
    plan = H.context_split_plan(whole.n_lo, whole.n_hi, R, window=w.window)
    assert plan[-1][2] <= whole.n_hi - w.window              # the window is on the last rank
    held = 0
    for part in plan:
        ws = H.workspace(256)
        pc = H.pack_kv_part(d["k"], d["v"], idx, w.window, part, bits, ws=ws, fmt=fmt)
        torch.cuda.synchronize()
        assert H.hq_read_device_status(ws) == 0
        assert pc.n_lo == part[1] - part[0] and pc.n_hi == part[3] - part[2]
        assert_pack_equal(cache_to_np(pc), _rows(wc, *part))
        held += pc.nbytes(with_pos=True)
    assert held == whole.nbytes(with_pos=True)               # each row is held by one rank


@pytest.mark.parametrize("bits,D", [(4, 128), (8, 64)])
def test_append_on_the_last_part(bits, D):
    """Tokens appended on the rank holding the window give the rows the
    whole cache's appends give; the merged decode after them matches the
    whole cache's decode."""
    H = hq()
    T = 70                                                   # > W: the ring wraps
    w = Workload("ap", "decode", 2, 8, 2, D, 3000 + T, 64, F5, bits, 800 + D + bits)
    x = make_inputs(w)
    d = to_dev(x)
    L0 = w.L - T
    k0, v0 = d["k"][:, :, :L0].contiguous(), d["v"][:, :, :L0].contiguous()
    kv0 = int(w.frac * L0)
    rng = np.random.default_rng(5)
    idx = torch.from_numpy(np.stack([[np.sort(rng.choice(L0 - w.window, kv0, replace=False))
                                      for _ in range(w.Hkv)] for _ in range(w.B)]).astype(np.int32)).cuda()
    n_lo0 = L0 - w.window - kv0
    whole = H.pack_kv(k0, v0, idx, w.window, bits, lo_cap=n_lo0 + T)
    R = 2
    plan = H.context_split_plan(n_lo0, kv0 + w.window, R, window=w.window)
    parts = [H.pack_kv_part(k0, v0, idx, w.window, p, bits,
                            lo_cap=(p[1] - p[0]) + (T if r == R - 1 else 0)) for r, p in enumerate(plan)]
    for t in range(T):
        kn = d["k"][:, :, L0 + t].contiguous()
        vn = d["v"][:, :, L0 + t].contiguous()
        H.kv_append(whole, kn, vn, L0 + t, w.window)
        H.kv_append_part(parts[-1], plan[-1], kn, vn, L0 + t, w.window, kv0)
    torch.cuda.synchronize()
    lo0, _, hi0, hi1 = plan[-1]
    wc = cache_to_np(whole)
    assert_pack_equal(cache_to_np(parts[-1]), _rows(wc, lo0, whole.n_lo, hi0, hi1))
    assert_pack_equal(cache_to_np(parts[0]), _rows(wc, *plan[0]))     # untouched
    outs, lses = zip(*[H.decode_attn(d["q"], p, w.Hkv, want_lse=True) for p in parts])
    out, lse = H.decode_merge(torch.stack(outs), torch.stack(lses))
    ref, ref_lse = H.decode_attn(d["q"], whole, w.Hkv, want_lse=True)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), ref.double().cpu().numpy(), "appended context split")
    assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=1e-4)


def _cp_gpu_worker(rank, world, port, q):
    """One rank, one process, on the one GPU, gloo between the processes
    (host-staged gathers; no kernel waits on another rank's): the probe over
    this rank's keys (probe_context_parallel), then this rank's part of the
    cache packed (pack_kv_part) and decoded with the exchange
    (decode_context_parallel)."""
    import datetime
    import os

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        H = hq()
        w = Workload("cp_gpu", "decode", 1, 8, 2, 128, 6000, 128, F5, 4, 4321)
        x = make_inputs(w)                       # the same seed on every rank: one context
        d = to_dev(x)
        off, n = H.probe_context_plan(w.L, world)[rank]
        idx = H.probe_context_parallel(d["q_probe"], d["k"][:, :, off:off + n].contiguous(), off,
                                       w.L, w.window, w.k_vert)
        n_lo, n_hi = w.n_lo, w.n_hi
        part = H.context_split_plan(n_lo, n_hi, world, window=w.window)[rank]
        # the oracle's index list drives the pack, so both sides hold one cache
        ridx = oracle.topk(oracle.probe_scores(x["q_probe"], x["k"], w.Hkv), w.window, w.k_vert)
        pc = H.pack_kv_part(d["k"], d["v"], torch.from_numpy(ridx).cuda(), w.window, part, w.bits)
        out, lse = H.decode_context_parallel(d["q"], pc, w.Hkv)
        torch.cuda.synchronize()
        q.put((rank, idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy(),
               pc.nbytes(), part))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_context_parallel_two_processes_end_to_end():
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_cp_gpu_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=280) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = Workload("cp_gpu", "decode", 1, 8, 2, 128, 6000, 128, F5, 4, 4321)
    x = make_inputs(w)
    sc = oracle.probe_scores(x["q_probe"], x["k"], w.Hkv)
    ridx = oracle.topk(sc, w.window, w.k_vert)
    ref = oracle.pack_kv(x["k"], x["v"], ridx, w.window, w.bits)
    full, full_lse = oracle.decode_attn(x["q"], ref, w.Hkv)
    total = 0
    for rank, idx, out, lse, nbytes, part in res:
        assert_index_sets(idx, ridx, sc, w.window)
        assert_close(out, full, f"decode_context_parallel rank {rank}")
        assert np.allclose(lse, full_lse, atol=1e-4, rtol=1e-5)
        total += nbytes
    # every rank holds about half of the cache
    assert all(abs(r[4] - total / world) <= 0.05 * total for r in res)
