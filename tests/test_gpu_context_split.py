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
