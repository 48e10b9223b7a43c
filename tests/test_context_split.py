"""Context-split decode (rows of one cache shared among ranks), host side.

The split plan is pure host logic; the merge of partial decodes is pinned by
the oracle: the decode of every row subset, merged by log-sum-exp weights,
equals the oracle's decode of the whole cache.  No GPU.
"""
import math

import numpy as np
import pytest

import oracle
from kv_cache_vertical_b200 import hq
from kv_cache_vertical_b200.synth import F5, Workload, make_inputs

RNG = np.random.default_rng(77)


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
def test_plan_covers_rows_once_and_balances_bytes(R):
    for n_lo, n_hi, D, bits in [(31002, 1766, 128, 4), (124000, 6600, 128, 8), (5000, 0, 64, 4),
                                (0, 300, 128, 4), (100, 5000, 128, 8), (777, 13, 64, 8)]:
        plan = hq.context_split_plan(n_lo, n_hi, R, D, bits)
        assert len(plan) == R
        assert [w for _, _, w in plan] == [False] * (R - 1) + [True]     # bf16 rows: last rank
        assert plan[0][0] == 0 and plan[-1][1] == n_lo
        for (a0, a1, _), (b0, b1, _) in zip(plan[:-1], plan[1:]):
            assert a1 == b0 and a0 <= a1                                # contiguous, disjoint
        for lo0, lo1, _ in plan:
            assert lo0 % 64 == 0                                        # aligned views
        b_lo, b_hi = 2 * (D * bits // 8 + D // 8), 4 * D
        load = [(lo1 - lo0) * b_lo + (n_hi * b_hi if w else 0) for lo0, lo1, w in plan]
        total = n_lo * b_lo + n_hi * b_hi
        if n_lo * b_lo >= 4 * R * 64 * b_lo and n_hi * b_hi <= total / R:
            assert max(load) <= total / R + 2 * 64 * b_lo


def _sub(c, lo0, lo1, with_hi):
    d = {n: np.ascontiguousarray(c[n][:, :, lo0:lo1]) for n in ("k_codes", "v_codes", "k_sz", "v_sz")}
    d["k_hi"] = c["k_hi"] if with_hi else c["k_hi"][:, :, :0]
    d["v_hi"] = c["v_hi"] if with_hi else c["v_hi"][:, :, :0]
    d.update(n_lo=lo1 - lo0, n_hi=c["n_hi"] if with_hi else 0, bits=c["bits"], group=c["group"],
             fmt=c.get("fmt", 0))
    return d


def merge_np(outs, lses):
    """Log-sum-exp merge written out (float64)."""
    lses = np.asarray(lses, np.float64)
    m = lses.max(0)
    w = np.exp(lses - m)
    out = (w[..., None] * np.asarray(outs, np.float64)).sum(0) / w.sum(0)[..., None]
    return out, m + np.log(w.sum(0))


@pytest.mark.parametrize("R,bits", [(2, 4), (3, 8), (4, 4)])
def test_merged_parts_equal_the_whole_cache(R, bits):
    w = Workload("cs", "decode", 2, 8, 2, 128, 3000, 128, F5, bits, 5 + R)
    x = make_inputs(w)
    c = oracle.pack_kv(x["k"], x["v"], x["planted"].numpy(), w.window, bits)
    full, full_lse = oracle.decode_attn(x["q"], c, w.Hkv)
    outs, lses = [], []
    for lo0, lo1, with_hi in hq.context_split_plan(c["n_lo"], c["n_hi"], R, w.D, bits):
        if lo1 - lo0 == 0 and not with_hi:
            outs.append(np.zeros_like(full))
            lses.append(np.full(full_lse.shape, -np.inf))
            continue
        o, l = oracle.decode_attn(x["q"], _sub(c, lo0, lo1, with_hi), w.Hkv)
        outs.append(o)
        lses.append(l)
    out, lse = merge_np(outs, lses)
    assert np.allclose(out, full, atol=1e-12, rtol=1e-10)
    assert np.allclose(lse, full_lse, atol=1e-12, rtol=1e-12)
    # a wrong split (a row range counted twice) is detected
    o2, l2 = oracle.decode_attn(x["q"], _sub(c, 0, 64, False), w.Hkv)
    bad, _ = merge_np(outs + [o2], lses + [l2])
    assert np.abs(bad - full).max() > 1e-6
