"""GPU parity of the hybrid prefill path: INT8 pre-pass and hybrid attention.

The index list comes from the oracle's probe (checked against the GPU probe
modulo ties); every expected value is the fp64 oracle's on the same inputs.
"""
import fractions

import numpy as np
import pytest
import torch

import oracle
from hq_testutil import assert_close, assert_index_sets, to_dev
from kv_cache_vertical_b200.synth import F5, WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


def oracle_idx(x, w: Workload):
    if w.k_vert == 0:
        return np.zeros((w.B, w.Hkv, 0), np.int32), None
    qp = x["q"][:, :, w.L - 64:].contiguous()
    sc = oracle.probe_scores(qp, x["k"], w.Hkv)
    return oracle.topk(sc, w.window, w.k_vert), sc


def run_prefill_case(w: Workload, rows=None, check_probe=True, fmt=0, planted_idx=False):
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    if planted_idx:
        # the seeded planted positions (sorted, distinct, before the window)
        # as the vertical set: no probe, so sequences shorter than the 64
        # probe queries work too
        ridx, rsc = x["planted"].numpy().astype(np.int32), None
        check_probe = False
    else:
        ridx, rsc = oracle_idx(x, w)
    if check_probe and w.k_vert > 0:
        gidx = H.probe_vertical(d["q"][:, :, w.L - 64:], d["k"], w.window, w.k_vert)
        torch.cuda.synchronize()
        assert_index_sets(gidx.cpu().numpy(), ridx, rsc, w.window)
    # INT8 pre-pass: bit-exact
    idx_d = torch.from_numpy(ridx).cuda()
    gq = [t.cpu().numpy() for t in H.prefill_quant(d["q"], d["k"], idx_d, fmt=fmt)]
    rq = oracle.prefill_quant(x["q"], x["k"], ridx, fmt=fmt)
    for g, r, name in zip(gq, rq, ("qi8", "sq", "ki8", "sk")):
        assert np.array_equal(g, r), f"{name} differs"
    out = H.prefill_attn(d["q"], d["k"], d["v"], idx_d, w.window, fmt=fmt)
    torch.cuda.synchronize()
    ref = oracle.prefill_attn(x["q"], x["k"], x["v"], ridx, w.window, quant=rq, rows=rows, fmt=fmt)
    g = out.cpu().numpy()
    if rows is not None:
        g = g[:, :, rows]
    return assert_close(g, ref, f"prefill {w.name}")


@pytest.mark.parametrize("G", [2, 4])
def test_prefill_small_ragged(G):
    w = Workload("p", "prefill", 1, 2 * G, 2, 128, 1000, 128, F5, 4, 11 + G)
    run_prefill_case(w)


def test_prefill_tensor_core_kernel_is_the_path():
    """The accepted shapes run the tcgen05 kernel (the query checks that the
    compiled kernel is usable on this device); the others are refused before
    any launch, never run on another kernel."""
    H = hq()
    for fmt in (0, 1):
        for G in (2, 4, 8):
            assert H.hq_prefill_supported(128, 8 * G, 8, fmt) == 0
        assert H.hq_prefill_supported(128, 8, 8, fmt) == 2          # one query head per KV head
        assert H.hq_prefill_supported(64, 4, 1, fmt) == 2           # head_dim 64
    for w in (Workload("g1", "prefill", 1, 2, 2, 128, 300, 32, F5, 4, 12),
              Workload("p64", "prefill", 2, 4, 1, 64, 700, 64, F5, 4, 21)):
        d = to_dev(make_inputs(w))
        idx = torch.from_numpy(make_inputs(w)["planted"].numpy()).cuda()
        with pytest.raises(H.HQError) as e:
            H.prefill_attn(d["q"], d["k"], d["v"], idx, w.window)
        assert e.value.status == 2


def test_prefill_window_larger_than_sequence():
    # everything is high precision: plain causal bf16 attention
    w = Workload("allhi", "prefill", 1, 2, 1, 128, 300, 400, fractions.Fraction(0), 4, 22)
    run_prefill_case(w, check_probe=False)


def test_prefill_no_window_no_vertical():
    # everything INT8
    w = Workload("alllo", "prefill", 1, 2, 1, 128, 513, 0, fractions.Fraction(0), 4, 23)
    run_prefill_case(w, check_probe=False)


def test_prefill_many_verticals_small_window():
    w = Workload("vert", "prefill", 1, 8, 1, 128, 1100, 16, fractions.Fraction(1, 4), 4, 24)
    run_prefill_case(w)


def test_prefill_medium_all_rows():
    w = Workload("med", "prefill", 1, 8, 2, 128, 4096, 128, F5, 4, 25)
    run_prefill_case(w)


@pytest.mark.slow
def test_prefill_full_size_sampled_rows():
    w = WORKLOADS["llama8b_prefill_32k"]
    rng = np.random.default_rng(5)
    N, W = w.L, w.window
    rows = np.unique(np.concatenate([
        np.arange(0, 8), np.arange(W - 4, W + 4), rng.integers(0, N, 48),
        np.arange(N - 64, N, 8), [N - 1]])).astype(np.int32)
    run_prefill_case(w, rows=rows)


def test_prefill_reports_bad_index_lists():
    """An index list that is not strictly ascending inside [0, N - window)
    sets HQ_DEV_BAD_INDEX in the workspace status word; a valid one does not.
    Every access stays in bounds either way (remaining-key positions are
    clamped by construction, vertical rows are gathered only when in range)."""
    H = hq()
    w = Workload("p", "prefill", 1, 4, 2, 128, 640, 128, F5, 4, 31)
    x = make_inputs(w)
    d = to_dev(x)
    ridx, _ = oracle_idx(x, w)
    ws = H.workspace(H.hq_prefill_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D, w.k_vert))
    good = torch.from_numpy(ridx).cuda()
    H.prefill_attn(d["q"], d["k"], d["v"], good, w.window, ws=ws)
    assert H.hq_read_device_status(ws) == 0
    for bad in (ridx[:, :, ::-1].copy(),                        # descending
                np.where(np.arange(w.k_vert) == 3, w.L - 1, ridx).astype(np.int32),  # in the window
                np.where(np.arange(w.k_vert) == 0, -5, ridx).astype(np.int32)):      # negative
        H.prefill_attn(d["q"], d["k"], d["v"], torch.from_numpy(bad).cuda(), w.window, ws=ws)
        assert H.hq_read_device_status(ws, clear=True) & H.HQ_DEV_BAD_INDEX
        assert H.hq_read_device_status(ws) == 0


# Short sequences on the tensor-core path (D = 128, two query heads per KV
# head): one, two or three 64-key tiles in all, lengths on and just past a
# tile edge, windows that are not a multiple of the tile, the diagonal-only
# window and no window.
SHORT = [(1, 16, 0), (37, 16, 20), (64, 0, 8), (65, 40, 16), (129, 64, 20), (200, 100, 4),
         (333, 1, 10)]


@pytest.mark.parametrize("N,W,inv_f", SHORT)
def test_prefill_short_sequences_tile_edges(N, W, inv_f):
    f = fractions.Fraction(1, inv_f) if inv_f else fractions.Fraction(0)
    w = Workload("short", "prefill", 1, 4, 2, 128, N, W, f, 4, 400 + N)
    run_prefill_case(w, planted_idx=True)


@pytest.mark.parametrize("N,W,inv_f", [(37, 16, 20), (129, 64, 20), (333, 1, 10)])
def test_prefill_fp8_short_sequences(N, W, inv_f):
    w = Workload("short_fp8", "prefill", 1, 4, 2, 128, N, W, fractions.Fraction(1, inv_f), 4, 500 + N)
    run_prefill_case(w, planted_idx=True, fmt=1)


# --------------------------------------------------------------------------
# FP8 (E4M3) low part, tcgen05 kind::f8f6f4
# --------------------------------------------------------------------------

@pytest.mark.parametrize("G", [2, 4, 8])
def test_prefill_fp8_small_ragged(G):
    w = Workload("p_fp8", "prefill", 1, 2 * G, 2, 128, 777, 64, F5, 4, 300 + G)
    run_prefill_case(w, fmt=1)


def test_prefill_fp8_medium_all_rows():
    w = Workload("p_fp8_med", "prefill", 2, 8, 2, 128, 2100, 128, F5, 4, 71)
    run_prefill_case(w, fmt=1)


def test_prefill_fp8_full_size_sampled_rows():
    w = WORKLOADS["llama8b_prefill_32k"]
    rows = np.array([0, 1, 127, 128, 4095, 16385, 32000, w.L - 1], np.int32)
    run_prefill_case(w, rows=rows, check_probe=False, fmt=1)


def test_prefill_fp8_rejected_off_the_tensor_core_path():
    H = hq()
    w = Workload("p_fp8_d64", "prefill", 1, 2, 1, 64, 256, 32, F5, 4, 1)
    d = to_dev(make_inputs(w))
    idx = torch.zeros(1, 1, 0, dtype=torch.int32, device="cuda")
    with pytest.raises(H.HQError):
        H.prefill_attn(d["q"], d["k"], d["v"], idx, w.window, fmt=1)
