"""GPU parity of the decode path: probe -> pack -> decode attention.

Every expected value comes from the fp64 oracle fed with the same seeded
inputs; the oracle's own index list drives both packs, so nothing the CUDA path
produces is ever an oracle input.
"""
import numpy as np
import pytest
import torch

import oracle
from hq_testutil import (assert_close, assert_index_sets, assert_pack_equal, cache_to_np, to_dev)
from kv_cache_vertical_b200.synth import F5, F25, WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


def run_decode_case(w: Workload, check_probe=True, planted_idx=False, fmt=0):
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    # probe (GPU) vs oracle; or, for large pack/decode cases, the seeded
    # planted positions (sorted, distinct, outside the window) as the list
    if planted_idx:
        ref_idx = x["planted"].numpy().astype(np.int32)
        check_probe = False
    else:
        ref_score = oracle.probe_scores(x["q_probe"], x["k"], w.Hkv)
        ref_idx = oracle.topk(ref_score, w.window, w.k_vert)
    if check_probe:
        gidx, gscore = H.probe_vertical(d["q_probe"], d["k"], w.window, w.k_vert, want_scores=True)
        torch.cuda.synchronize()
        gs = gscore.cpu().numpy()
        G, P = w.G, 64
        assert np.allclose(gs, ref_score, rtol=1e-3, atol=1e-6 * G * P), \
            f"probe scores: max rel {np.max(np.abs(gs - ref_score) / (np.abs(ref_score) + 1e-9)):.2e}"
        assert_index_sets(gidx.cpu().numpy(), ref_idx, ref_score, w.window)
    # pack with the oracle's index list on both sides: bit-exact
    idx_d = torch.from_numpy(ref_idx).cuda()
    ws = H.workspace(256)
    cache = H.pack_kv(d["k"], d["v"], idx_d, w.window, w.bits, ws=ws, fmt=fmt)
    ref_cache = oracle.pack_kv(x["k"], x["v"], ref_idx, w.window, w.bits, 32, fmt)
    torch.cuda.synchronize()
    assert H.hq_read_device_status(ws) == 0
    assert_pack_equal(cache_to_np(cache), ref_cache)
    # decode on identical quantized inputs
    out, lse = H.decode_attn(d["q"], cache, w.Hkv, want_lse=True)
    ref_out, ref_lse = oracle.decode_attn(x["q"], ref_cache, w.Hkv)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), ref_out, f"decode {w.name}")
    assert np.allclose(lse.cpu().numpy(), ref_lse, atol=1e-4, rtol=1e-5)
    return out, ref_out


def test_tiny_decode_config():
    run_decode_case(WORKLOADS["tiny_decode"])


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_ragged_multi_tile(bits, G):
    # L not a multiple of any tile, several splits, both code widths
    w = Workload("ragged", "decode", 2, 2 * G, 2, 128, 5003, 128, F5, bits, 77 + G)
    run_decode_case(w)


@pytest.mark.parametrize("D", [64, 128])
def test_decode_head_dims(D):
    w = Workload("hd", "decode", 1, 4, 2, D, 2100, 64, F25, 4, 99)
    run_decode_case(w)


def test_decode_edge_nothing_low():
    # k_vert = L - W: the low segment is empty, decode is plain bf16 attention
    w = Workload("nolow", "decode", 1, 4, 1, 128, 600, 100, F5, 4, 5)
    w = w.replace(frac=__import__("fractions").Fraction(500, 600))
    assert w.n_lo == 0
    run_decode_case(w, check_probe=True)


def test_decode_edge_nothing_high():
    # no window and no vertical columns: everything is low-bit
    w = Workload("nohi", "decode", 1, 2, 1, 128, 777, 0, __import__("fractions").Fraction(0), 4, 6)
    assert w.n_hi == 0
    run_decode_case(w, check_probe=False)


def test_decode_short_context():
    w = Workload("short", "decode", 3, 8, 2, 128, 70, 16, F5, 8, 8)
    run_decode_case(w)


def test_pack_reports_bad_index_lists():
    H = hq()
    w = Workload("bad", "decode", 1, 2, 1, 64, 300, 32, F5, 4, 9)
    x = to_dev(make_inputs(w))
    idx = torch.arange(w.k_vert, dtype=torch.int32, device="cuda").view(1, 1, -1).contiguous()
    idx[0, 0, 3] = idx[0, 0, 2]                 # repeated entry
    ws = H.workspace(256)
    H.pack_kv(x["k"], x["v"], idx, w.window, 4, ws=ws)
    assert H.hq_read_device_status(ws, clear=True) & H.HQ_DEV_BAD_INDEX
    assert H.hq_read_device_status(ws) == 0
    idx = torch.arange(w.k_vert, dtype=torch.int32, device="cuda").view(1, 1, -1) + 290  # >= L - W
    H.pack_kv(x["k"], x["v"], idx.contiguous(), w.window, 4, ws=ws)
    assert H.hq_read_device_status(ws) & H.HQ_DEV_BAD_INDEX


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_many_tiles_per_cta(bits):
    # 32 (b, kv head) pairs over the SMs: every CTA streams many tiles through
    # its shared-memory ring, so every stage and barrier phase is reused
    w = Workload("multitile", "decode", 4, 32, 8, 128, 20000, 128, F5, bits, 31)
    run_decode_case(w, planted_idx=True)


def test_decode_more_pairs_than_a_join_search_covers():
    # 384 (b, kv head) pairs, more than the 256 a CTA looks through when it
    # joins another pair (the search wraps around the pair index), with a
    # ragged context so that the last tile of every pair is partial
    w = Workload("manypairs", "decode", 48, 16, 8, 128, 2011, 64, F5, 4, 41)
    assert w.B * w.Hkv > 256
    run_decode_case(w, planted_idx=True)


def test_llama8b_decode_full_size():
    run_decode_case(WORKLOADS["llama8b_decode_32k"])


def _full_size_sampled(w: Workload, samples, fmt=0):
    """Run probe / pack / decode at full size in the benchmark's launch
    configuration; compare the sampled (b, kv head) slices with the oracle."""
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    idx = H.probe_vertical(d["q_probe"], d["k"], w.window, w.k_vert)
    cache = H.pack_kv(d["k"], d["v"], idx, w.window, w.bits, fmt=fmt)
    out = H.decode_attn(d["q"], cache, w.Hkv)
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    gc = cache_to_np(cache)
    gout = out.cpu().numpy()
    G = w.G
    for b, h in samples:
        qs = x["q"][b:b + 1, h * G:(h + 1) * G].contiguous()
        qp = x["q_probe"][b:b + 1, h * G:(h + 1) * G].contiguous()
        ks, vs = x["k"][b:b + 1, h:h + 1].contiguous(), x["v"][b:b + 1, h:h + 1].contiguous()
        sc = oracle.probe_scores(qp, ks, 1)
        ridx = oracle.topk(sc, w.window, w.k_vert)
        assert_index_sets(gidx[b:b + 1, h:h + 1], ridx, sc, w.window)
        rc = oracle.pack_kv(ks, vs, ridx, w.window, w.bits, 32, fmt)
        ro, _ = oracle.decode_attn(qs, rc, 1)
        if np.array_equal(gidx[b:b + 1, h:h + 1], ridx):
            sc_np = {k: (v[b:b + 1, h:h + 1] if isinstance(v, np.ndarray) else None)
                     for k, v in gc.items()}
            so = gout[b:b + 1, h * G:(h + 1) * G]
        else:
            # a tie swapped members of the set: pack and decode this slice on
            # the GPU with the oracle's list, so it is still compared exactly
            c1 = H.pack_kv(ks.cuda(), vs.cuda(), torch.from_numpy(ridx).cuda(), w.window, w.bits,
                           fmt=fmt)
            so = H.decode_attn(qs.cuda(), c1, 1).cpu().numpy()
            sc_np = cache_to_np(c1)
        assert_pack_equal(sc_np, rc)
        assert_close(so, ro, f"{w.name} b={b} h={h}")


@pytest.mark.slow
def test_batched_decode_int4_full_size():
    _full_size_sampled(WORKLOADS["batched_decode_128k_int4"], [(0, 0), (7, 5)])


@pytest.mark.slow
def test_batched_decode_int8_full_size():
    _full_size_sampled(WORKLOADS["batched_decode_128k_int8"], [(3, 2), (6, 7)])


@pytest.mark.slow
def test_70b_decode_full_size():
    _full_size_sampled(WORKLOADS["70b_decode_64k"], [(0, 0), (31, 7), (17, 3)])


# --------------------------------------------------------------------------
# FP8 (E4M3) low-bit format
# --------------------------------------------------------------------------

@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_fp8_ragged(G, D):
    # codes and scales bit-exact, decode within tolerance; ragged L, several
    # tiles per CTA on both lines
    w = Workload("fp8", "decode", 2, 2 * G, 2, D, 5003, 128, F5, 8, 177 + G + D)
    run_decode_case(w, fmt=1)


def test_decode_fp8_many_tiles_per_cta():
    w = Workload("fp8_multitile", "decode", 4, 32, 8, 128, 20000, 128, F5, 8, 41)
    run_decode_case(w, planted_idx=True, fmt=1)


def test_llama8b_decode_fp8_full_size():
    w = WORKLOADS["llama8b_decode_32k"].replace(bits=8)
    run_decode_case(w, fmt=1)


@pytest.mark.slow
def test_batched_decode_fp8_full_size():
    w = WORKLOADS["batched_decode_128k_int8"]
    _full_size_sampled(w, [(1, 4), (5, 0)], fmt=1)
