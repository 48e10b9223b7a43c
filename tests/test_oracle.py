"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a library
routine (numpy / torch float64), brute force on tiny inputs, a closed form, an
invariant, or a figure printed on the pages (tests/golden/).  The cases are
chosen so that a dropped term, a wrong sign or index, an off-by-one in the
window or causal mask, or a transposed operand fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_vertical_b200.synth import Workload, F5, make_inputs

RNG = np.random.default_rng(1234)


def bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def f64(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.float64)


# --------------------------------------------------------------------------
# 16-bit formats
# --------------------------------------------------------------------------

def test_bf16_widening_matches_torch_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(p)) for p in pats[::7]])
    r = ref[::7]
    ok = np.isnan(r) == np.isnan(got)
    assert ok.all()
    assert np.array_equal(got[~np.isnan(r)], r[~np.isnan(r)])


def test_f16_widening_matches_numpy_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(p)) for p in pats])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])


def test_f16_rounding_matches_numpy():
    xs = [0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25,
          3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 * (1 - 2.0 ** -12), 1.0 + 2.0 ** -11,
          1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0, -7.5e-5]
    xs += list(RNG.standard_normal(20000) * 10.0 ** RNG.integers(-8, 5, 20000))
    # exact binary16 midpoints (ties) must go to even
    lo = np.arange(1, 31000, 37, dtype=np.uint16)
    mids = (lo.view(np.float16).astype(np.float64) + (lo + 1).view(np.float16).astype(np.float64)) / 2
    xs += list(mids) + list(-mids)
    for x in xs:
        with np.errstate(over="ignore"):
            want = int(np.array([x], np.float64).astype(np.float16).view(np.uint16)[0])
        got = oracle.f64_to_f16(float(x))
        assert got == want, (x, hex(got), hex(want))


# --------------------------------------------------------------------------
# Quantizer (KV pack)
# --------------------------------------------------------------------------

def _unpack(packed: np.ndarray, bits: int, D: int) -> np.ndarray:
    if bits == 8:
        return packed.astype(np.int64)
    out = np.zeros(D, np.int64)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out


def _sz(sz: np.ndarray):
    v = sz.view(np.float16).astype(np.float64)
    return v[0::2], v[1::2]


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_closed_form_power_of_two_grid(bits):
    qmax = (1 << bits) - 1
    for trial in range(50):
        s = 2.0 ** int(RNG.integers(-6, -1))
        # bf16 holds 8 significant bits: keep every grid point an exact integer * s
        mn = s * int(RNG.integers(-40, 40) if bits == 4 else RNG.integers(-128, 1))
        c = RNG.integers(0, qmax + 1, 32)
        i0, i1 = RNG.choice(32, 2, replace=False)
        c[i0], c[i1] = 0, qmax
        x = mn + c * s
        xb = bf16(x)
        assert np.array_equal(f64(xb).numpy(), x), "grid must be exact in bf16"
        packed, sz = oracle.quant_row(xb, bits, 32)
        scales, zeros = _sz(sz)
        assert scales[0] == s and zeros[0] == mn + 0.0
        assert np.array_equal(_unpack(packed, bits, 32), c)


def test_quant_constant_group_gives_zero_codes():
    for val in (0.0, 1.5, -3.25, 60.0):
        packed, sz = oracle.quant_row(bf16(np.full(32, val)), 4, 32)
        s, z = _sz(sz)
        assert s[0] == 0.0 and z[0] == val
        assert not packed.any()
        assert np.float16(val).view(np.uint16) == sz[1] or val == 0.0


def test_quant_ties_round_to_even_and_nibble_order():
    # s = (15 - 0) / 15 = 1, z = 0: 2.5 -> 2, 3.5 -> 4, 0.5 -> 0, 14.5 -> 14
    x = np.zeros(32)
    x[1] = 15.0
    x[2], x[3], x[4], x[5] = 2.5, 3.5, 0.5, 14.5
    x[6] = 1.0
    packed, sz = oracle.quant_row(bf16(x), 4, 32)
    c = _unpack(packed, 4, 32)
    assert list(c[:7]) == [0, 15, 2, 4, 0, 14, 1]
    # even channel in the low nibble: byte 0 holds channels 0 (low) and 1 (high)
    assert packed[0] == 0x00 | (15 << 4)
    assert packed[3] == 1  # channels 6 (code 1) and 7 (code 0)


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_round_trip_bound(bits):
    qmax = (1 << bits) - 1
    x = RNG.standard_normal((200, 128)) * RNG.choice([0.01, 1.0, 10.0], (200, 1))
    xb = bf16(x)
    for r in range(200):
        packed, sz = oracle.quant_row(xb[r], bits, 32)
        c = _unpack(packed, bits, 128)
        s, z = _sz(sz)
        xv = f64(xb[r]).numpy()
        for g in range(4):
            seg = xv[32 * g:32 * g + 32]
            cg = c[32 * g:32 * g + 32]
            assert cg.min() >= 0 and cg.max() <= qmax
            # s and z are the fp16 roundings of the exact range / qmax and minimum
            assert s[g] == float(np.float16((seg.max() - seg.min()) / qmax))
            assert z[g] == float(np.float16(seg.min()))
            xh = s[g] * cg + z[g]
            inside = (seg >= z[g]) & (seg <= z[g] + qmax * s[g])
            assert np.all(np.abs(xh - seg)[inside] <= s[g] / 2 * (1 + 1e-12))
            # outside the representable range the code is clamped to the nearest end
            assert np.all(cg[seg < z[g]] == 0) and np.all(cg[seg > z[g] + qmax * s[g]] == qmax)


# --------------------------------------------------------------------------
# FP8 (E4M3) low-bit format
# --------------------------------------------------------------------------

def _e4m3_torch(codes) -> np.ndarray:
    """Decode E4M3 bytes with torch's float8_e4m3fn (library routine)."""
    t = torch.as_tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_decode_all_codes_matches_torch():
    ref = _e4m3_torch(np.arange(256))
    got = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2        # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_encode_round_trip_ties_and_saturation():
    vals = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert oracle.f64_to_e4m3(vals[c]) == c, c                        # exact values
    pos = [c for c in range(0x7F)]                                        # 0 .. 448 ascending
    for lo_c, hi_c in zip(pos[:-1], pos[1:]):
        mid = (vals[lo_c] + vals[hi_c]) / 2                               # ties: even code
        assert oracle.f64_to_e4m3(mid) == (lo_c if lo_c % 2 == 0 else hi_c)
        assert oracle.f64_to_e4m3(-mid) == 0x80 | (lo_c if lo_c % 2 == 0 else hi_c)
        assert oracle.f64_to_e4m3(np.nextafter(mid, 0)) == lo_c
        assert oracle.f64_to_e4m3(np.nextafter(mid, 1e9)) == hi_c
    for v in (448.0, 460.0, 464.0, 480.0, 1e6, np.inf):                   # satfinite
        assert oracle.f64_to_e4m3(v) == 0x7E and oracle.f64_to_e4m3(-v) == 0xFE
    assert oracle.f64_to_e4m3(-0.0) == 0x80 and oracle.f64_to_e4m3(-1e-9) == 0x80
    # in range, RNE agrees with torch's float32 -> float8_e4m3fn cast
    x = (RNG.standard_normal(20000) * RNG.choice([1e-3, 0.1, 1.0, 50.0], 20000)).astype(np.float32)
    x = x[np.abs(x) < 440]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f64_to_e4m3(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def _fp8_row(xb):
    packed, sz = oracle.quant_row(xb, 8, 32, oracle.FMT_FP8)
    s = np.array([float(np.frombuffer(np.uint16(b).tobytes(), np.float16)[0]) for b in sz[0::2]])
    z = sz[1::2]
    return packed, s, z


def test_fp8_quant_closed_forms():
    # power-of-two scale: values that are E4M3 numbers times 2^-3, with the
    # group maximum 448 * 2^-3, quantize exactly
    codes = RNG.integers(0, 0x7E, 32).astype(np.uint8) | (RNG.integers(0, 2, 32).astype(np.uint8) << 7)
    codes[5] = 0x7E
    x = _e4m3_torch(codes) * 2.0 ** -3
    packed, s, z = _fp8_row(bf16(np.concatenate([x, x, x, x])))
    assert np.all(s == 2.0 ** -3) and np.all(z == 0)
    got = _e4m3_torch(packed[:32])
    assert np.array_equal(got * s[0], x)
    # constant group: every code is 448 (or -448), the scale is fp16(|c| / 448)
    for val in (1.0, -3.25, 1e-3):
        packed, s, z = _fp8_row(bf16(np.full(128, val)))
        assert np.all(packed == (0x7E if val > 0 else 0xFE))
        assert np.all(s == float(np.float16(abs(float(bf16([val])[0])) / 448)))
    # zero group: scale 0, codes 0
    packed, s, z = _fp8_row(bf16(np.zeros(128)))
    assert np.all(packed == 0) and np.all(s == 0)


def test_fp8_quant_round_trip_bound():
    x = RNG.standard_normal((200, 128)) * RNG.choice([0.01, 1.0, 10.0], (200, 1))
    xb = bf16(x)
    for r in range(200):
        packed, s, z = _fp8_row(xb[r])
        xv = f64(xb[r]).numpy()
        xh = _e4m3_torch(packed) * np.repeat(s, 32)
        for g in range(4):
            seg, hg = xv[32 * g:32 * g + 32], xh[32 * g:32 * g + 32]
            amax = np.abs(seg).max()
            assert s[g] == float(np.float16(amax / 448))
            # half a unit of the 3-bit mantissa, or of the subnormal spacing,
            # plus the saturation slack of a rounded-down scale
            bound = np.maximum(np.abs(hg) * 2.0 ** -4, s[g] * 2.0 ** -10) + amax * 2.0 ** -10
            assert np.all(np.abs(hg - seg) <= bound * (1 + 1e-12))
            assert np.all(np.sign(hg) * np.sign(seg) >= 0)


# --------------------------------------------------------------------------
# Probe (column sums) and top-k
# --------------------------------------------------------------------------

def _probe_ref(qp, k, Hkv, scale):
    """torch float64 softmax over the causal probe rows, summed per column."""
    B, Hq, P, D = qp.shape
    L = k.shape[2]
    G = Hq // Hkv
    out = torch.zeros(B, Hkv, L, dtype=torch.float64)
    pos = torch.arange(L - P, L)
    mask = torch.arange(L)[None, :] > pos[:, None]
    for b in range(B):
        for h in range(Hq):
            s = f64(qp[b, h]) @ f64(k[b, h // G]).T * scale
            s = s.masked_fill(mask, -math.inf)
            out[b, h // G] += torch.softmax(s, dim=-1).sum(0)
    return out.numpy()


def test_probe_scores_match_torch_softmax():
    B, Hq, Hkv, P, L, D = 2, 4, 2, 16, 90, 32
    qp = bf16(RNG.standard_normal((B, Hq, P, D)))
    k = bf16(RNG.standard_normal((B, Hkv, L, D)) * 2)
    sc = 1 / math.sqrt(D)
    got = oracle.probe_scores(qp, k, Hkv, sc)
    ref = _probe_ref(qp, k, Hkv, sc)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
    # each softmax row sums to one: the columns sum to G * P per KV head
    assert np.allclose(got.sum(-1), (Hq // Hkv) * P, rtol=1e-12)
    # keys after the last probe row are never seen; the last key only by the last row
    assert got[..., L - 1].min() > 0 and np.all(got[..., L - P:].sum() > 0)


def test_probe_hand_case_picks_the_attended_key():
    D, L, P, W = 64, 300, 64, 16
    u = np.zeros(D)
    u[5] = 1.0
    k = np.zeros((1, 1, L, D))
    k[0, 0, 137] = 3 * u                            # the only key aligned with the queries
    k[0, 0, :, 40] = RNG.standard_normal(L) * 0.01  # orthogonal noise
    qp = np.tile(2 * u, (1, 2, P, 1)) + np.pad(RNG.standard_normal((1, 2, P, 1)) * 0.1,
                                                ((0, 0), (0, 0), (0, 0), (40, D - 41)))
    score = oracle.probe_scores(bf16(qp), bf16(k), 1)
    idx = oracle.topk(score, W, 1)
    assert idx[0, 0, 0] == 137


def test_topk_brute_force_with_ties():
    for trial in range(30):
        L, W = int(RNG.integers(20, 200)), int(RNG.integers(0, 20))
        kv = int(RNG.integers(0, L - W + 1))
        # few distinct values -> many exact ties
        s = RNG.integers(0, 6, (2, 3, L)).astype(np.float64) / 4
        idx = oracle.topk(s, W, kv)
        for b in range(2):
            for h in range(3):
                cand = np.arange(L - W)
                order = np.lexsort((cand, -s[b, h, :L - W]))  # score desc, then index asc
                want = np.sort(cand[order[:kv]])
                assert np.array_equal(idx[b, h], want)
                assert np.all(idx[b, h] < L - W)          # disjoint from the window


# --------------------------------------------------------------------------
# Pack: partition invariants and row contents
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_pack_partition_and_rows(bits):
    B, Hkv, L, D, W = 2, 2, 300, 64, 32
    kv = 20
    k = bf16(RNG.standard_normal((B, Hkv, L, D)))
    v = bf16(RNG.standard_normal((B, Hkv, L, D)))
    idx = np.sort(np.stack([np.stack([RNG.choice(L - W, kv, replace=False) for _ in range(Hkv)])
                            for _ in range(B)]), -1).astype(np.int32)
    c = oracle.pack_kv(k, v, idx, W, bits, 32)
    kb, vb = oracle.bits(k), oracle.bits(v)
    for b in range(B):
        for h in range(Hkv):
            lo = c["lo_pos"][b, h]
            allpos = np.concatenate([lo, idx[b, h], np.arange(L - W, L)])
            assert np.array_equal(np.sort(allpos), np.arange(L))       # exact partition
            assert np.all(np.diff(lo) > 0)                              # ascending, compacted
            win = np.arange(L - W, L)
            hi_src = np.concatenate([idx[b, h], win[np.argsort(win % W)]])   # ring: row kv + p mod W
            assert np.array_equal(c["k_hi"][b, h], kb[b, h, hi_src])
            assert np.array_equal(c["v_hi"][b, h], vb[b, h, hi_src])
            for r in (0, len(lo) // 2, len(lo) - 1):
                pk, szk = oracle.quant_row(k[b, h, lo[r]], bits, 32)
                assert np.array_equal(c["k_codes"][b, h, r], pk)
                assert np.array_equal(c["k_sz"][b, h, r].reshape(-1), szk)


# --------------------------------------------------------------------------
# Decode cache maintenance: append = pack of the longer prefix
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits,D,W,fmt", [(4, 64, 32, 0), (8, 64, 32, 0), (4, 128, 7, 0),
                                         (8, 128, 0, 0), (8, 128, 16, 1)])
def test_append_equals_pack_of_longer_prefix(bits, D, W, fmt):
    """Packing L0 tokens and appending tokens L0 .. L0+t-1 one by one gives the
    cache packed from L0 + t tokens with the same vertical set, field for
    field: the evicted position, its low row, lo_pos, the ring slot and the
    quantizer all have to be right for that.  t > W so the ring wraps."""
    B, Hkv, L0, t, kv = 2, 2, 150, 45, 9
    k = bf16(RNG.standard_normal((B, Hkv, L0 + t, D)) * 2.0)
    v = bf16(RNG.standard_normal((B, Hkv, L0 + t, D)))
    idx = np.sort(np.stack([np.stack([RNG.choice(L0 - W, kv, replace=False) for _ in range(Hkv)])
                            for _ in range(B)]), -1).astype(np.int32)
    c = oracle.pack_kv(k[:, :, :L0], v[:, :, :L0], idx, W, bits, 32, fmt)
    for L in range(L0, L0 + t):
        c = oracle.kv_append(c, k[:, :, L], v[:, :, L], L, W)
    ref = oracle.pack_kv(k, v, idx, W, bits, 32, fmt)
    assert c["n_lo"] == ref["n_lo"] and c["n_hi"] == ref["n_hi"]
    for name in ("k_codes", "v_codes", "k_sz", "v_sz", "k_hi", "v_hi", "lo_pos"):
        assert np.array_equal(c[name], ref[name]), name


def test_append_moves_exactly_one_token():
    """One append: the window row kv + L mod W now holds token L, the old
    occupant (position L - W) is the new last low row, quantized by the row
    quantizer, and nothing else changed."""
    B, Hkv, L, D, W, kv = 1, 3, 200, 64, 16, 11
    k = bf16(RNG.standard_normal((B, Hkv, L + 1, D)))
    v = bf16(RNG.standard_normal((B, Hkv, L + 1, D)))
    idx = np.sort(np.stack([np.stack([RNG.choice(L - W, kv, replace=False) for _ in range(Hkv)])
                            for _ in range(B)]), -1).astype(np.int32)
    c0 = oracle.pack_kv(k[:, :, :L], v[:, :, :L], idx, W, 4, 32)
    c1 = oracle.kv_append(c0, k[:, :, L], v[:, :, L], L, W)
    kb, vb = oracle.bits(k), oracle.bits(v)
    slot = kv + L % W
    for h in range(Hkv):
        assert np.array_equal(c1["k_hi"][0, h, slot], kb[0, h, L])
        assert np.array_equal(c1["v_hi"][0, h, slot], vb[0, h, L])
        assert np.array_equal(c0["k_hi"][0, h, slot], kb[0, h, L - W])      # the evicted token
        others = np.arange(kv + W) != slot
        assert np.array_equal(c1["k_hi"][0, h, others], c0["k_hi"][0, h, others])
        assert c1["lo_pos"][0, h, -1] == L - W
        assert np.array_equal(c1["lo_pos"][0, h, :-1], c0["lo_pos"][0, h])
        pk, szk = oracle.quant_row(k[0, h, L - W], 4, 32)
        assert np.array_equal(c1["k_codes"][0, h, -1], pk)
        assert np.array_equal(c1["k_sz"][0, h, -1].reshape(-1), szk)
        pv, szv = oracle.quant_row(v[0, h, L - W], 4, 32)
        assert np.array_equal(c1["v_codes"][0, h, -1], pv)
        assert np.array_equal(c1["v_sz"][0, h, -1].reshape(-1), szv)


def test_memory_overhead_matches_the_pages():
    """+15% non-window cache at 5% retention vs strict 4-bit (golden, cited)."""
    txt = open(__file__.replace("test_oracle.py", "golden/memory_overhead.txt")).read()
    want = float([l for l in txt.splitlines() if l.startswith("overhead")][0].split("=")[1])
    L, W, D = 32768, 128, 128
    w = Workload("m", "decode", 1, 1, 1, D, L, W, F5)
    bits_hybrid = w.n_lo * D * 4 + w.k_vert * D * 16        # code / bf16 payload only
    bits_strict = (L - W) * D * 4
    got = bits_hybrid / bits_strict - 1
    assert abs(got - want) < 0.005


# --------------------------------------------------------------------------
# Decode attention
# --------------------------------------------------------------------------

def _sdpa(q, k, v, scale, causal=False):
    return torch.nn.functional.scaled_dot_product_attention(
        f64(q), f64(k), f64(v), is_causal=causal, scale=scale)


def test_decode_all_high_precision_equals_exact_attention():
    # k_vert = L - W: nothing is quantized, so hybrid attention is exact attention
    B, Hq, Hkv, L, D, W = 2, 4, 2, 96, 64, 16
    k = bf16(RNG.standard_normal((B, Hkv, L, D)) * 2)
    v = bf16(RNG.standard_normal((B, Hkv, L, D)))
    q = bf16(RNG.standard_normal((B, Hq, D)))
    idx = np.tile(np.arange(L - W, dtype=np.int32), (B, Hkv, 1))
    c = oracle.pack_kv(k, v, idx, W)
    assert c["n_lo"] == 0
    out, lse = oracle.decode_attn(q, c, Hkv)
    G = Hq // Hkv
    kk = k.repeat_interleave(G, dim=1)
    vv = v.repeat_interleave(G, dim=1)
    ref = _sdpa(q[:, :, None], kk, vv, 1 / math.sqrt(D))[:, :, 0]
    assert np.allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bhd,bhld->bhl", f64(q), f64(kk)) / math.sqrt(D)
    assert np.allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def _dequant_np(codes, sz, bits, D):
    n = codes.shape[0]
    if bits == 8:
        c = codes.astype(np.float64)
    else:
        c = np.zeros((n, D))
        c[:, 0::2] = codes & 0xF
        c[:, 1::2] = codes >> 4
    s = sz[..., 0].view(np.float16).astype(np.float64)
    z = sz[..., 1].view(np.float16).astype(np.float64)
    return c * np.repeat(s, 32, axis=1) + np.repeat(z, 32, axis=1)


@pytest.mark.parametrize("bits,fmt", [(4, 0), (8, 0), (8, 1)])
def test_decode_matches_dequantize_then_attend(bits, fmt):
    w = Workload("t", "decode", 2, 4, 2, 64, 256, 32, F5, bits, 7)
    x = make_inputs(w)
    sc = oracle.probe_scores(x["q_probe"], x["k"], w.Hkv)
    idx = oracle.topk(sc, w.window, w.k_vert)
    c = oracle.pack_kv(x["k"], x["v"], idx, w.window, bits, 32, fmt)
    dq = _dequant_np if fmt == 0 else (lambda codes, sz, bits_, D: _dequant_fp8_np(codes, sz, D))
    out, lse = oracle.decode_attn(x["q"], c, w.Hkv)
    for b in range(w.B):
        for h in range(w.Hq):
            kh = h // w.G
            kd = np.concatenate([dq(c["k_codes"][b, kh], c["k_sz"][b, kh], bits, w.D),
                                 f64(x["k"][b, kh][np.concatenate(
                                     [idx[b, kh], np.arange(w.L - w.window, w.L)])]).numpy()])
            vd = np.concatenate([dq(c["v_codes"][b, kh], c["v_sz"][b, kh], bits, w.D),
                                 f64(x["v"][b, kh][np.concatenate(
                                     [idx[b, kh], np.arange(w.L - w.window, w.L)])]).numpy()])
            qd = f64(x["q"][b, h]).numpy()
            p = torch.softmax(torch.from_numpy(kd @ qd / math.sqrt(w.D)), 0).numpy()
            assert abs(p.sum() - 1) < 1e-12
            assert np.allclose(out[b, h], p @ vd, atol=1e-12)
    # quantization moves the result away from exact attention (the outlier
    # channels stretch the per-group grids), 8-bit much less than 4-bit
    kk = x["k"].repeat_interleave(w.G, 1)
    vv = x["v"].repeat_interleave(w.G, 1)
    exact = _sdpa(x["q"][:, :, None], kk, vv, 1 / math.sqrt(w.D))[:, :, 0].numpy()
    err = np.abs(out - exact).mean()
    assert 0 < err < (0.5 if bits == 4 else 0.05)


def _dequant_fp8_np(codes, sz, D):
    """s * e4m3(c) with torch's float8 decoding and numpy float16 scales."""
    s = np.asarray(sz).reshape(codes.shape[0], D // 32, 2)[..., 0].view(np.float16).astype(np.float64)
    return _e4m3_torch(codes) * np.repeat(s, 32, axis=1)


# --------------------------------------------------------------------------
# Prefill: INT8 pre-pass and hybrid attention
# --------------------------------------------------------------------------

def test_prefill_quant_matches_numpy_float32():
    B, Hq, Hkv, N, D = 1, 2, 1, 160, 64
    q = bf16(RNG.standard_normal((B, Hq, N, D)) * 3)
    k = bf16(RNG.standard_normal((B, Hkv, N, D)))
    idx = np.array([[[2, 5, 70, 71, 100]]], np.int32)      # vertical columns (never quantized)
    rem = np.setdiff1d(np.arange(N), idx[0, 0])             # remaining keys, position order
    k[0, 0, rem[64:128]] = 0                                 # an all-zero block -> scale 1, codes 0
    k[0, 0, 70] = 1000.0                                     # a huge vertical key must not widen any scale
    qi8, sq, ki8, sk = oracle.prefill_quant(q, k, idx, 64)
    assert ki8.shape == (B, Hkv, N - 5, D) and sk.shape == (B, Hkv, 3)
    qf = q.float().numpy()
    amax = np.abs(qf).max(-1)
    assert np.array_equal(sq, (amax / np.float32(127)).astype(np.float32))
    want = np.clip(np.rint(qf / sq[..., None]), -127, 127)
    assert np.array_equal(qi8, want.astype(np.int8))
    kf = k.float().numpy()[0, 0][rem]
    for blk in range(3):
        seg = kf[64 * blk:64 * blk + 64]
        a = np.abs(seg).max()
        s = np.float32(1) if a == 0 else np.float32(a) / np.float32(127)
        assert sk[0, 0, blk] == s
        assert np.array_equal(ki8[0, 0, 64 * blk:64 * blk + 64],
                              np.clip(np.rint(seg / s), -127, 127).astype(np.int8))
    assert np.abs(qi8).max() == 127 and sk[0, 0, 1] == 1 and not ki8[0, 0, 64:128].any()
    assert sk.max() < 1000.0 / 127


def test_prefill_fp8_quant_matches_float32_and_torch_cast():
    """FP8 low part: s = fl32(amax / 448), c = E4M3(fl32(x / s)) -- numpy
    float32 for the divisions, torch's float8_e4m3fn cast (nearest even) for
    the last rounding; vertical keys never quantized, zero blocks scale 1."""
    B, Hq, Hkv, N, D = 1, 2, 1, 160, 64
    q = bf16(RNG.standard_normal((B, Hq, N, D)) * 3)
    k = bf16(RNG.standard_normal((B, Hkv, N, D)))
    idx = np.array([[[2, 5, 70, 71, 100]]], np.int32)
    rem = np.setdiff1d(np.arange(N), idx[0, 0])
    k[0, 0, rem[64:128]] = 0
    k[0, 0, 70] = 1000.0
    qc, sq, kc, sk = oracle.prefill_quant(q, k, idx, 64, fmt=oracle.FMT_FP8)

    def e4m3(x32):          # float32 quotients, all within +-448 (1 + 2^-23)
        x32 = np.clip(x32, -448, 448)
        return torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.int8).numpy()
    qf = q.float().numpy()
    assert np.array_equal(sq, (np.abs(qf).max(-1) / np.float32(448)).astype(np.float32))
    assert np.array_equal(qc, e4m3((qf / sq[..., None]).astype(np.float32)))
    kf = k.float().numpy()[0, 0][rem]
    for blk in range(3):
        seg = kf[64 * blk:64 * blk + 64]
        a = np.abs(seg).max()
        sblk = np.float32(1) if a == 0 else np.float32(a) / np.float32(448)
        assert sk[0, 0, blk] == sblk
        assert np.array_equal(kc[0, 0, 64 * blk:64 * blk + 64], e4m3((seg / sblk).astype(np.float32)))
    assert sk[0, 0, 1] == 1 and not kc[0, 0, 64:128].any()
    assert np.abs(_e4m3_torch(qc.view(np.uint8))).max() == 448      # the row maximum maps to 448


def test_prefill_fp8_path_is_exact_on_e4m3_inputs():
    # rows and blocks whose maximum is 448 get scale 1 and codes equal to the
    # values when the values are E4M3 numbers: the all-low FP8 path is then
    # exact attention on those values
    B, Hq, Hkv, N, D = 1, 2, 1, 128, 16
    vals = _e4m3_torch(np.arange(0, 0x60, 3).astype(np.uint8))       # 0 .. 96, exact in bf16
    vals = np.concatenate([vals, -vals])
    q = RNG.choice(vals, (B, Hq, N, D))
    k = RNG.choice(vals, (B, Hkv, N, D))
    q[..., 0] = 448
    k[..., 0, :] = 0
    k[..., 0, 1] = 448
    k[..., 64, 1] = -448
    v = RNG.standard_normal((B, Hkv, N, D))
    scale = 1 / 2 ** 18
    out = oracle.prefill_attn(bf16(q), bf16(k), bf16(v), np.zeros((B, Hkv, 0), np.int32),
                              window=0, scale=scale, fmt=oracle.FMT_FP8)
    ref = _sdpa(bf16(q), bf16(k).repeat_interleave(2, 1), bf16(v).repeat_interleave(2, 1),
                scale, True)
    assert np.allclose(out, ref.numpy(), atol=1e-12)
    # and the INT8 reading of the same inputs is not exact (its grid is coarser)
    out8 = oracle.prefill_attn(bf16(q), bf16(k), bf16(v), np.zeros((B, Hkv, 0), np.int32),
                               window=0, scale=scale)
    assert np.abs(out8 - ref.numpy()).max() > 1e-9


def test_prefill_all_high_precision_equals_causal_attention():
    B, Hq, Hkv, N, D = 1, 4, 2, 70, 32
    q = bf16(RNG.standard_normal((B, Hq, N, D)))
    k = bf16(RNG.standard_normal((B, Hkv, N, D)))
    v = bf16(RNG.standard_normal((B, Hkv, N, D)))
    idx = np.zeros((B, Hkv, 0), np.int32)
    out = oracle.prefill_attn(q, k, v, idx, window=N)
    ref = _sdpa(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), 1 / math.sqrt(D), True)
    assert np.allclose(out, ref.numpy(), atol=1e-12)


def test_prefill_int8_path_is_exact_on_integer_inputs():
    # rows / blocks whose amax is 127 get scale 1 and codes equal to the values,
    # so the all-low INT8 path must equal exact attention on those integers
    B, Hq, Hkv, N, D = 1, 2, 1, 128, 16
    q = RNG.integers(-3, 4, (B, Hq, N, D)).astype(np.float64)
    k = RNG.integers(-3, 4, (B, Hkv, N, D)).astype(np.float64)
    q[..., 0] = 127
    k[..., 0, :] = 0
    k[..., 0, 1] = 127
    k[..., 64, 1] = -127
    v = RNG.standard_normal((B, Hkv, N, D))
    scale = 1 / 4096
    out = oracle.prefill_attn(bf16(q), bf16(k), bf16(v), np.zeros((B, Hkv, 0), np.int32),
                              window=0, scale=scale)
    ref = _sdpa(bf16(q), bf16(k).repeat_interleave(2, 1), bf16(v).repeat_interleave(2, 1),
                scale, True)
    assert np.allclose(out, ref.numpy(), atol=1e-12)


def test_prefill_mixed_pairs_follow_window_and_vertical_sets():
    """Per-pair precision: window wins, verticals are high, everything else INT8."""
    B, Hq, Hkv, N, D, W = 1, 2, 1, 200, 32, 24
    q = bf16(RNG.standard_normal((B, Hq, N, D)) * 2)
    k = bf16(RNG.standard_normal((B, Hkv, N, D)) * 2)
    v = bf16(RNG.standard_normal((B, Hkv, N, D)))
    idx = np.array([[[3, 50, 51, 120, 170]]], np.int32)
    quant = oracle.prefill_quant(q, k, idx)
    qi8, sq, ki8, sk = quant
    rows = np.array([0, 1, 23, 24, 25, 50, 74, 75, 120, 143, 144, 145, 199], np.int32)
    out = oracle.prefill_attn(q, k, v, idx, W, quant=quant, rows=rows)
    sc = 1 / math.sqrt(D)
    vert = set(idx[0, 0].tolist())
    for h in range(Hq):
        for ri, i in enumerate(rows):
            logits = np.empty(i + 1)
            for j in range(i + 1):
                if i - j < W or j in vert:
                    logits[j] = float(f64(q[0, h, i]) @ f64(k[0, 0, j])) * sc
                else:
                    c = j - int((idx[0, 0] < j).sum())   # rank among the remaining keys
                    dot = int(np.dot(qi8[0, h, i].astype(np.int64), ki8[0, 0, c].astype(np.int64)))
                    logits[j] = dot * float(sq[0, h, i]) * float(sk[0, 0, c // 64]) * sc
            p = torch.softmax(torch.from_numpy(logits), 0).numpy()
            ref = p @ f64(v[0, 0, :i + 1]).numpy()
            assert np.allclose(out[0, h, ri], ref, atol=1e-12), (h, i)
    # moving the window by one key changes rows whose boundary key is low-bit
    out2 = oracle.prefill_attn(q, k, v, idx, W + 1, quant=quant, rows=rows)
    assert np.abs(out2 - out)[:, :, rows >= W + 1].max() > 1e-9
