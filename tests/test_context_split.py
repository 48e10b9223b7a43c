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
        plan = hq.context_split_plan(n_lo, n_hi, R)
        assert len(plan) == R
        assert plan[0][0] == 0 and plan[-1][1] == n_lo and plan[0][2] == 0 and plan[-1][3] == n_hi
        for a, b in zip(plan[:-1], plan[1:]):
            assert a[1] == b[0] and a[3] == b[2]                        # contiguous, disjoint
        for lo0, lo1, hi0, hi1 in plan:
            assert lo0 <= lo1 and hi0 <= hi1 and lo0 % 64 == 0          # aligned views
        b_lo, b_hi = 2 * (D * bits // 8 + D // 8), 4 * D
        load = [(lo1 - lo0) * b_lo + (hi1 - hi0) * b_hi for lo0, lo1, hi0, hi1 in plan]
        total = n_lo * b_lo + n_hi * b_hi
        assert max(load) <= total / R + 64 * b_lo + b_hi                # equal shares


def _sub(c, lo0, lo1, hi0, hi1):
    d = {n: np.ascontiguousarray(c[n][:, :, lo0:lo1]) for n in ("k_codes", "v_codes", "k_sz", "v_sz")}
    d["k_hi"] = np.ascontiguousarray(c["k_hi"][:, :, hi0:hi1])
    d["v_hi"] = np.ascontiguousarray(c["v_hi"][:, :, hi0:hi1])
    d.update(n_lo=lo1 - lo0, n_hi=hi1 - hi0, bits=c["bits"], group=c["group"],
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
    for part in hq.context_split_plan(c["n_lo"], c["n_hi"], R):
        if part[1] == part[0] and part[3] == part[2]:
            outs.append(np.zeros_like(full))
            lses.append(np.full(full_lse.shape, -np.inf))
            continue
        o, l = oracle.decode_attn(x["q"], _sub(c, *part), w.Hkv)
        outs.append(o)
        lses.append(l)
    out, lse = merge_np(outs, lses)
    assert np.allclose(out, full, atol=1e-12, rtol=1e-10)
    assert np.allclose(lse, full_lse, atol=1e-12, rtol=1e-12)
    # a wrong split (a row range counted twice) is detected
    o2, l2 = oracle.decode_attn(x["q"], _sub(c, 0, 64, 0, 0), w.Hkv)
    bad, _ = merge_np(outs + [o2], lses + [l2])
    assert np.abs(bad - full).max() > 1e-6


# ---------------------------------------------------------------------------
# Context-split probe: the context's keys shared among ranks
# ---------------------------------------------------------------------------

def _f64(t):
    return t.float().numpy().astype(np.float64) if hasattr(t, "numpy") else np.asarray(t, np.float64)


def probe_shard_np(q_probe, k_shard, key_off, L, Hkv, stats=None):
    """One rank's part of the probe, restated from the definition (fp64):
    without `stats`, each probe row's (max, Z = sum of exp(s - max)) over the
    rank's visible keys; with the context's stats, the rank's column scores.
    Probe row p sits at context position L - P + p and sees keys j <= it."""
    q, k = _f64(q_probe), _f64(k_shard)
    B, Hq, P, D = q.shape
    Ls, G = k.shape[2], Hq // Hkv
    pos = L - P + np.arange(P)
    vis = (key_off + np.arange(Ls))[None, :] <= pos[:, None]               # [P, Ls]
    s = np.einsum("bhpd,bhld->bhpl", q, np.repeat(k, G, axis=1)) / math.sqrt(D)
    s = np.where(vis[None, None], s, -np.inf)
    if stats is None:
        m = s.max(axis=3)
        z = np.where(np.isfinite(m), np.exp(s - np.where(np.isfinite(m), m, 0)[..., None]).sum(axis=3), 0.0)
        return m, z                                                        # [B, Hq, P]
    m, z = stats
    w = np.exp(s - m[..., None]) / z[..., None]
    return w.reshape(B, Hkv, G * P, Ls).sum(axis=2)                       # [B, Hkv, Ls]


def merge_stats_np(parts):
    ms = np.stack([m for m, _ in parts])
    zs = np.stack([z for _, z in parts])
    m = ms.max(axis=0)
    return m, (zs * np.exp(np.where(np.isfinite(ms), ms - m, -np.inf))).sum(axis=0)


def shard_candidates_np(score, key_off, L, window, k_vert):
    """A rank's best k_vert candidates (context positions before L - window),
    ordered by (score desc, position asc), -1 padded."""
    B, Hkv, Ls = score.shape
    ncand = max(0, min(Ls, L - window - key_off))
    ci = np.full((B, Hkv, k_vert), -1, np.int64)
    cs = np.full((B, Hkv, k_vert), -np.inf)
    for b in range(B):
        for h in range(Hkv):
            order = sorted(range(ncand), key=lambda j: (-score[b, h, j], j))[:k_vert]
            ci[b, h, :len(order)] = np.array(order, np.int64) + key_off
            cs[b, h, :len(order)] = score[b, h, order]
    return ci, cs


def merge_candidates_np(cis, css, L, window, k_vert):
    dense = np.full(cis[0].shape[:2] + (L - window,), -np.inf)
    for ci, cs in zip(cis, css):
        for b in range(ci.shape[0]):
            for h in range(ci.shape[1]):
                for j, v in zip(ci[b, h], cs[b, h]):
                    if j >= 0:
                        dense[b, h, j] = v
    return oracle.topk(np.pad(dense, ((0, 0), (0, 0), (0, window)), constant_values=-np.inf),
                       window, k_vert)


@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_probe_plan_and_split_equal_the_whole_context(R):
    w = Workload("pcp", "decode", 1, 8, 2, 64, 700, 64, F5, 4, 900 + R)
    x = make_inputs(w)
    qp, k = x["q_probe"], x["k"]
    plan = hq.probe_context_plan(w.L, R)
    assert plan[0][0] == 0 and sum(n for _, n in plan) == w.L
    assert all(a[0] + a[1] == b[0] for a, b in zip(plan[:-1], plan[1:]))
    assert max(n for _, n in plan) - min(n for _, n in plan) <= 1
    parts = [probe_shard_np(qp, k[:, :, o:o + n], o, w.L, w.Hkv) for o, n in plan]
    stats = merge_stats_np(parts)
    score = np.concatenate([probe_shard_np(qp, k[:, :, o:o + n], o, w.L, w.Hkv, stats)
                            for o, n in plan], axis=2)
    full = oracle.probe_scores(qp, k, w.Hkv)
    assert np.allclose(score, full, rtol=1e-12, atol=1e-15)
    cand = [shard_candidates_np(score[:, :, o:o + n], o, w.L, w.window, w.k_vert) for o, n in plan]
    idx = merge_candidates_np([c[0] for c in cand], [c[1] for c in cand], w.L, w.window, w.k_vert)
    assert np.array_equal(idx, oracle.topk(full, w.window, w.k_vert))


def test_probe_plan_with_more_ranks_than_keys():
    # ranks beyond the keys get empty ranges; the ranges still tile [0, L)
    for L, R in [(3, 5), (1, 2), (7, 7), (10, 3)]:
        plan = hq.probe_context_plan(L, R)
        assert len(plan) == R and sum(n for _, n in plan) == L
        pos = [o + i for o, n in plan for i in range(n)]
        assert pos == list(range(L))
        assert sum(1 for _, n in plan if n == 0) == max(0, R - L)
