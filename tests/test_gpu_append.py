"""GPU parity of decode cache maintenance: pack -> append tokens -> decode.

The expected cache after appending tokens L0 .. L0+t-1 to a cache packed from
L0 tokens is the oracle's pack of all L0 + t tokens with the same vertical set
(the CPU suite pins the oracle's append chain to exactly that); the expected
decode output is the oracle's decode over that cache.  The vertical set is the
seeded planted positions that fall before the prefix's window, so no value the
CUDA path produces is ever an oracle input.
"""
import numpy as np
import pytest
import torch

import oracle
from hq_testutil import assert_close, assert_pack_equal, cache_to_np, to_dev
from kv_cache_vertical_b200.synth import F5, Workload, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


def prefix_vertical_set(planted: np.ndarray, limit: int) -> np.ndarray:
    """The first k planted positions below `limit` of every (b, kv head), k the
    smallest such count over the heads (one k for the whole cache)."""
    B, Hkv, _ = planted.shape
    below = [[planted[b, h][planted[b, h] < limit] for h in range(Hkv)] for b in range(B)]
    k = min(len(x) for row in below for x in row)
    return np.ascontiguousarray(np.array([[x[:k] for x in row] for row in below], np.int32))


def run_append_case(w: Workload, t: int, check_steps=(), decode_steps=(), fmt=0):
    """Pack the first L0 = w.L - t tokens, append the other t one by one on the
    GPU, then compare the cache and a decode against the oracle."""
    H = hq()
    x = make_inputs(w)
    d = to_dev(x)
    L0, W = w.L - t, w.window
    idx = prefix_vertical_set(x["planted"].numpy(), L0 - W)
    kv = idx.shape[2]
    n_lo0 = L0 - W - kv
    cache = H.pack_kv(d["k"][:, :, :L0].contiguous(), d["v"][:, :, :L0].contiguous(),
                      torch.from_numpy(idx).cuda(), W, w.bits, lo_cap=n_lo0 + t, fmt=fmt)
    ref = oracle.pack_kv(x["k"][:, :, :L0], x["v"][:, :, :L0], idx, W, w.bits, 32, fmt)
    for s in range(t):
        L = L0 + s
        H.kv_append(cache, d["k"][:, :, L].contiguous(), d["v"][:, :, L].contiguous(), L, W)
        ref = oracle.kv_append(ref, x["k"][:, :, L], x["v"][:, :, L], L, W)
        if s in check_steps:
            torch.cuda.synchronize()
            assert_pack_equal(cache_to_np(cache), ref)
        if s in decode_steps:
            out = H.decode_attn(d["q"], cache, w.Hkv)
            ref_out, _ = oracle.decode_attn(x["q"], ref, w.Hkv)
            torch.cuda.synchronize()
            assert_close(out.cpu().numpy(), ref_out, f"decode after append {s}")
    torch.cuda.synchronize()
    assert cache.n_lo == n_lo0 + t
    got = cache_to_np(cache)
    assert_pack_equal(got, ref)
    # the appended cache is the pack of the whole sequence
    full = oracle.pack_kv(x["k"], x["v"], idx, W, w.bits, 32, fmt)
    assert_pack_equal(got, full)
    out, lse = H.decode_attn(d["q"], cache, w.Hkv, want_lse=True)
    ref_out, ref_lse = oracle.decode_attn(x["q"], full, w.Hkv)
    torch.cuda.synchronize()
    assert_close(out.cpu().numpy(), ref_out, f"decode {w.name}")
    assert np.allclose(lse.cpu().numpy(), ref_lse, atol=1e-4, rtol=1e-5)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_append_chain_ring_wraps(bits, D):
    # t > W: the window ring wraps; B, Hkv > 1; ragged lengths
    w = Workload("append", "decode", 2, 8, 2, D, 1537 + 90, 64, F5, bits, 311 + D + bits)
    run_append_case(w, t=90, check_steps=(0, 1, 63, 64), decode_steps=(0, 40))


def test_append_no_window():
    # W = 0: each new token is quantized straight into the low segment
    w = Workload("append_w0", "decode", 1, 4, 2, 128, 900 + 20, 0, F5, 4, 17)
    run_append_case(w, t=20, check_steps=(0,), decode_steps=(5,))


@pytest.mark.parametrize("G", [1, 8])
def test_append_decode_loop(G):
    # the decode loop: every step appends then attends; the low segment grows
    # across a tile boundary of the decode (the tile plan changes on the way)
    w = Workload("loop", "decode", 1, 2 * G, 2, 128, 2000 + 40, 128, F5, 4, 5 + G)
    run_append_case(w, t=40, decode_steps=tuple(range(0, 40, 3)))


def test_llama8b_append_full_size():
    # Llama-3.1-8B-shaped layer at the 32K decode context: 32 query / 8 KV
    # heads, D = 128, W = 128, INT4; the last 16 tokens arrive by append
    w = Workload("llama8b_append_32k", "decode", 1, 32, 8, 128, 32768, 128, F5, 4, 2024)
    run_append_case(w, t=16, check_steps=(0,))


@pytest.mark.parametrize("D", [64, 128])
def test_append_fp8(D):
    w = Workload("append_fp8", "decode", 2, 8, 2, D, 1300 + 70, 64, F5, 8, 91 + D)
    run_append_case(w, t=70, check_steps=(0, 64), decode_steps=(3,), fmt=1)
