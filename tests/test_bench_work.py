"""Host logic of the benchmark: the algorithmic work every roofline figure is
divided by.  Decode bytes are checked against the per-configuration figures
worked out from the cache layout (codes + fp16 scale/zero per 32 channels +
bf16 rows + q + fp32 out); the prefill's pair counts against a brute-force
classification of every causal pair."""
import numpy as np
import pytest

import bench
from kv_cache_vertical_b200.synth import WORKLOADS, make_inputs


@pytest.mark.parametrize("name,mbytes", [
    ("llama8b_decode_32k", 46.94),
    ("batched_decode_128k_int4", 1492.9),
    ("batched_decode_128k_int8", 2511.9),
    ("70b_decode_64k", 2856.6),
])
def test_decode_bytes_per_configuration(name, mbytes):
    w = WORKLOADS[name]
    got = bench.decode_bytes(w.B, w.Hq, w.Hkv, w.D, w.n_lo, w.n_hi, w.bits) / 1e6
    assert abs(got - mbytes) <= 0.01 * mbytes / 10 + 0.01, (name, got)


def test_decode_bytes_by_hand():
    # one (b, kv head), D = 64, INT4: a low row is 32 B of codes + 2 groups x
    # (s, z) fp16 = 8 B, for K and V; a bf16 row is 128 B, for K and V
    got = bench.decode_bytes(1, 2, 1, 64, 10, 3, 4)
    assert got == 10 * 2 * (32 + 8) + 3 * 2 * 128 + 2 * 64 * 2 + 2 * 64 * 4


def _brute_pairs(idx, N, W):
    """(low, hi) causal pair counts per (b, kv head) by classifying every pair."""
    out = []
    for row in idx.reshape(idx.shape[0] * idx.shape[1], idx.shape[2]):
        vert = np.zeros(N, bool)
        vert[row] = True
        low = hi = 0
        for i in range(N):
            for j in range(i + 1):
                if j > i - W or (vert[j] and j <= i - W):
                    hi += 1
                else:
                    low += 1
        out.append((low, hi))
    return out


@pytest.mark.parametrize("N,W", [(1, 4), (37, 16), (300, 64), (301, 0)])
def test_prefill_work_matches_brute_force(N, W):
    w = WORKLOADS["llama8b_prefill_32k"].replace(L=N, window=W, Hq=4, Hkv=2)
    idx = make_inputs(w)["planted"].numpy()
    i8, bf = bench.prefill_work(idx, N, W, w.D, w.Hq, w.Hkv)
    G = w.Hq // w.Hkv
    total = N * (N + 1) // 2
    low = sum(lo for lo, _ in _brute_pairs(idx, N, W))
    hi = sum(h for _, h in _brute_pairs(idx, N, W))
    nbh = idx.shape[0] * idx.shape[1]
    assert i8 == 2 * w.D * G * low
    assert bf == 2 * w.D * G * (nbh * total + hi)       # P.V over every pair + hi QK


def test_prefill_window_closed_form():
    # the closed form used for long sequences equals the explicit sum
    for N, W in [(5000, 128), (4096, 4096), (4100, 1)]:
        explicit = sum(min(i + 1, W) for i in range(N))
        closed = W * (W + 1) // 2 + (N - W) * W if N >= W else N * (N + 1) // 2
        assert explicit == closed


def test_prefill_work_full_size_magnitudes():
    # the 32K layer with its planted vertical set: about 4.15 T INT8 ops and
    # 4.65 T bf16 flops (the vertical pairs depend on where the columns sit)
    w = WORKLOADS["llama8b_prefill_32k"]
    idx = make_inputs(w)["planted"].numpy()
    i8, bf = bench.prefill_work(idx, w.L, w.window, w.D, w.Hq, w.Hkv)
    assert abs(i8 / 1e12 - 4.15) < 0.05 and abs(bf / 1e12 - 4.65) < 0.05
