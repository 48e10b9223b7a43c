"""GPU parity of the vertical-line probe across the shapes its tensor-core
passes treat differently: probe-row counts P that are not multiples of 8 or
16 (zero-filled padding rows), one, two, four and eight query heads per KV
head (one, one, two and four 128-row blocks; the eight-head case splits the
column sums into row groups and the row statistics into 64-key sub-tiles),
head_dim 64, contexts shorter than one 128-key tile and ragged tails, a
probe-row count equal to the context, and a caller head stride (the last P
rows of a longer query block).  The expected values are the fp64 oracle's;
scores within 1e-3 relative, index sets equal except where the oracle's own
scores tie within 1e-5 of the k-th."""
import fractions

import numpy as np
import pytest
import torch

import oracle
from hq_testutil import assert_index_sets
from kv_cache_vertical_b200.synth import F5, Workload, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


def check_probe(w: Workload, P: int):
    H = hq()
    x = make_inputs(w)
    qp = x["q_probe"][:, :, 64 - P:].contiguous()     # the P most recent probe rows
    k = x["k"]
    ref_score = oracle.probe_scores(qp, k, w.Hkv)
    ref_idx = oracle.topk(ref_score, w.window, w.k_vert)
    gidx, gscore = H.probe_vertical(qp.cuda(), k.cuda(), w.window, w.k_vert, want_scores=True)
    torch.cuda.synchronize()
    gs = gscore.cpu().numpy()
    rel = np.abs(gs - ref_score) / (np.abs(ref_score) + 1e-30)
    assert np.all((rel <= 1e-3) | (np.abs(gs - ref_score) <= 1e-6 * w.G * P)), f"max rel {rel.max():.2e}"
    assert_index_sets(gidx.cpu().numpy(), ref_idx, ref_score, w.window)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("P", [1, 7, 13, 40, 64])
def test_probe_rows_and_groups(G, P):
    w = Workload("pr", "decode", 1, 2 * G, 2, 128, 3001, 128, F5, 4, 600 + 7 * G + P)
    check_probe(w, P)


@pytest.mark.parametrize("L", [64, 100, 128, 129, 1000])
def test_probe_short_contexts_head_dim_64(L):
    w = Workload("ps", "decode", 2, 4, 2, 64, L, 16, fractions.Fraction(1, 10), 4, 700 + L)
    check_probe(w, min(64, L))


def test_probe_head_stride_of_a_query_block():
    # the last 64 rows of [B, Hq, N, D] prefill queries: head stride N * D
    H = hq()
    w = Workload("pq", "prefill", 1, 8, 2, 128, 2500, 128, F5, 4, 777)
    x = make_inputs(w)
    q = x["q"].cuda()
    qp_view = q[:, :, w.L - 64:]
    assert qp_view.stride(1) == w.L * w.D
    gidx, gscore = H.probe_vertical(qp_view, x["k"].cuda(), w.window, w.k_vert, want_scores=True)
    qp = x["q"][:, :, w.L - 64:].contiguous()
    ref_score = oracle.probe_scores(qp, x["k"], w.Hkv)
    torch.cuda.synchronize()
    assert np.allclose(gscore.cpu().numpy(), ref_score, rtol=1e-3, atol=1e-6 * 256)
    assert_index_sets(gidx.cpu().numpy(), oracle.topk(ref_score, w.window, w.k_vert), ref_score, w.window)


def test_topk_on_exact_ties():
    # many exactly equal scores: the k columns are the lowest-index ties
    H = hq()
    B, Hkv, L, W, k = 2, 3, 40000, 128, 2000
    rng = np.random.default_rng(9)
    s = rng.integers(0, 50, size=(B, Hkv, L)).astype(np.float32) / 64.0
    s[0, 1, :] = 0.25                                  # every candidate ties
    ref = oracle.topk(s.astype(np.float64), W, k)
    # the merge entry point scatters R ranks' candidates (k per rank) into one
    # score row per pair and runs the top-k kernel: give it every candidate
    ncand = L - W
    R = (ncand + k - 1) // k
    ci = np.full((R, B, Hkv, k), -1, np.int32)
    cs = np.full((R, B, Hkv, k), -np.finfo(np.float32).max, np.float32)
    for r in range(R):
        j = np.arange(r * k, min((r + 1) * k, ncand))
        ci[r, :, :, :j.size] = j
        cs[r, :, :, :j.size] = s[:, :, j]
    idx = torch.empty(B, Hkv, k, dtype=torch.int32, device="cuda")
    ws = H.workspace(H.hq_probe_merge_workspace_size(B, Hkv, L, W))
    H.hq_probe_merge_topk(torch.from_numpy(ci).cuda(), torch.from_numpy(cs).cuda(), R, B, Hkv, L, W,
                          k, idx, ws)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ref)
