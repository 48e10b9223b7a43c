"""fp64 CPU oracle for HyQuant hybrid-precision attention (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or runs it, and shares no code with
it.  The arithmetic lives in ``hq_oracle.c``; this module only compiles it
with gcc and marshals numpy arrays through ctypes.

16-bit floating-point tensors are passed as raw bit patterns (numpy uint16);
use :func:`bits` to view a torch bf16/fp16 CPU tensor that way.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.hqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.hqo_bf16_to_f64.restype = D
        lib.hqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.hqo_f16_to_f64.restype = D
        lib.hqo_f64_to_f16.argtypes = [D]
        lib.hqo_f64_to_f16.restype = ctypes.c_uint16
        lib.hqo_probe_scores.argtypes = [P, P, I, I, I, I, I, I, D, P]
        lib.hqo_topk.argtypes = [P, I, I, I, I, I, P]
        lib.hqo_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.hqo_e4m3_to_f64.restype = D
        lib.hqo_f64_to_e4m3.argtypes = [D]
        lib.hqo_f64_to_e4m3.restype = ctypes.c_uint8
        lib.hqo_quant_row.argtypes = [P, I, I, I, I, P, P]
        lib.hqo_pack_kv.argtypes = [P, P, P] + [I] * 9 + [P] * 7
        lib.hqo_kv_append.argtypes = [P, P] + [I] * 11 + [P] * 7
        lib.hqo_decode_attn.argtypes = [P] * 7 + [I] * 9 + [D, P, P]
        lib.hqo_prefill_quant.argtypes = [P, P, P] + [I] * 8 + [P] * 4
        lib.hqo_prefill_attn.argtypes = [P] * 8 + [I] * 9 + [D, P, I, P]
        lib.hqo_max_threads.argtypes = []
        for f in ("hqo_probe_scores", "hqo_topk", "hqo_quant_row", "hqo_pack_kv", "hqo_kv_append",
                  "hqo_decode_attn", "hqo_prefill_quant", "hqo_prefill_attn", "hqo_max_threads"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    return np.ascontiguousarray(bits(a))


def bits(t) -> np.ndarray:
    """View a 16-bit tensor / array as its uint16 bit patterns (no rounding)."""
    if isinstance(t, np.ndarray):
        return t.view(np.uint16) if t.dtype != np.uint16 else t
    import torch
    t = t.detach().cpu().contiguous()
    assert t.element_size() == 2, "expected a 16-bit tensor"
    return t.view(torch.int16).numpy().view(np.uint16)


def max_threads() -> int:
    return _load().hqo_max_threads()


def bf16_to_f64(b: int) -> float:
    return _load().hqo_bf16_to_f64(b)


def f16_to_f64(h: int) -> float:
    return _load().hqo_f16_to_f64(h)


def f64_to_f16(x: float) -> int:
    return _load().hqo_f64_to_f16(x)


def default_scale(D: int) -> float:
    return 1.0 / float(np.sqrt(D))


def probe_scores(q_probe, k, Hkv: int, scale: float | None = None) -> np.ndarray:
    """Column sums of causal softmax weights of the probe rows, fp64 [B, Hkv, L]."""
    qp, kk = _u16(q_probe), _u16(k)
    B, Hq, P, D = qp.shape
    L = kk.shape[2]
    out = np.zeros((B, Hkv, L), np.float64)
    rc = _load().hqo_probe_scores(_p(qp), _p(kk), B, Hq, Hkv, P, L, D,
                                  default_scale(D) if scale is None else scale, _p(out))
    assert rc == 0, rc
    return out


def topk(score: np.ndarray, window: int, kv: int) -> np.ndarray:
    """Top-kv columns of [0, L - window): (score desc, index asc), returned ascending."""
    s = np.ascontiguousarray(score, np.float64)
    B, Hkv, L = s.shape
    idx = np.zeros((B, Hkv, kv), np.int32)
    rc = _load().hqo_topk(_p(s), B, Hkv, L, window, kv, _p(idx))
    assert rc == 0, rc
    return idx


FMT_INT, FMT_FP8 = 0, 1      # low-bit code formats: asymmetric integer, FP8 E4M3


def e4m3_to_f64(c: int) -> float:
    return _load().hqo_e4m3_to_f64(int(c))


def f64_to_e4m3(v: float) -> int:
    return _load().hqo_f64_to_e4m3(float(v))


def quant_row(x, bits_: int = 4, group: int = 32, fmt: int = FMT_INT):
    """Quantize one row of bf16 values -> (packed codes u8, interleaved (s, z) f16 bits)."""
    xb = _u16(x).reshape(-1)
    D = xb.shape[0]
    packed = np.zeros(D * bits_ // 8, np.uint8)
    sz = np.zeros(2 * (D // group), np.uint16)
    rc = _load().hqo_quant_row(_p(xb), D, bits_, group, fmt, _p(packed), _p(sz))
    assert rc == 0, rc
    return packed, sz


def pack_kv(k, v, idx, window: int, bits_: int = 4, group: int = 32, fmt: int = FMT_INT) -> dict:
    """Build the hybrid cache (canonical layout) from bf16 K, V [B, Hkv, L, D]."""
    kk, vv = _u16(k), _u16(v)
    B, Hkv, L, D = kk.shape
    idx = np.ascontiguousarray(idx, np.int32)
    kv = idx.shape[2]
    n_lo, n_hi = L - window - kv, kv + window
    rb, ng = D * bits_ // 8, D // group
    out = dict(
        k_codes=np.zeros((B, Hkv, n_lo, rb), np.uint8),
        v_codes=np.zeros((B, Hkv, n_lo, rb), np.uint8),
        k_sz=np.zeros((B, Hkv, n_lo, ng, 2), np.uint16),
        v_sz=np.zeros((B, Hkv, n_lo, ng, 2), np.uint16),
        k_hi=np.zeros((B, Hkv, n_hi, D), np.uint16),
        v_hi=np.zeros((B, Hkv, n_hi, D), np.uint16),
        lo_pos=np.zeros((B, Hkv, n_lo), np.int32),
    )
    rc = _load().hqo_pack_kv(_p(kk), _p(vv), _p(idx), B, Hkv, L, D, window, kv, bits_, group, fmt,
                             _p(out["k_codes"]), _p(out["v_codes"]), _p(out["k_sz"]),
                             _p(out["v_sz"]), _p(out["k_hi"]), _p(out["v_hi"]), _p(out["lo_pos"]))
    assert rc == 0, rc
    out.update(n_lo=n_lo, n_hi=n_hi, bits=bits_, group=group, fmt=fmt)
    return out


def kv_append(cache: dict, k_new, v_new, L: int, window: int) -> dict:
    """One decode step of cache maintenance: token L (bf16 K/V [B, Hkv, D])
    enters the window ring, position L - W leaves it for the low segment.
    Returns a new cache dict with n_lo + 1 low rows; ``cache`` is not changed."""
    kn, vn = _u16(k_new), _u16(v_new)
    B, Hkv, D = kn.shape
    n_lo, n_hi = int(cache["n_lo"]), int(cache["n_hi"])
    kv = n_hi - window
    out = {}
    for name in ("k_codes", "v_codes", "k_sz", "v_sz", "lo_pos"):
        a = np.asarray(cache[name])
        grown = np.zeros((B, Hkv, n_lo + 1) + a.shape[3:], a.dtype)
        grown[:, :, :n_lo] = a[:, :, :n_lo]
        out[name] = grown
    out["k_hi"] = np.array(cache["k_hi"], np.uint16, copy=True)
    out["v_hi"] = np.array(cache["v_hi"], np.uint16, copy=True)
    rc = _load().hqo_kv_append(
        _p(kn), _p(vn), B, Hkv, D, L, window, kv, int(cache["bits"]), int(cache["group"]),
        int(cache.get("fmt", FMT_INT)), n_lo, n_lo + 1, _p(out["k_codes"]), _p(out["v_codes"]), _p(bits(out["k_sz"])),
        _p(bits(out["v_sz"])), _p(out["k_hi"]), _p(out["v_hi"]), _p(out["lo_pos"]))
    assert rc == 0, rc
    out.update(n_lo=n_lo + 1, n_hi=n_hi, bits=cache["bits"], group=cache["group"],
               fmt=cache.get("fmt", FMT_INT))
    return out


def decode_attn(q, cache: dict, Hkv: int, scale: float | None = None):
    """Exact fp64 decode attention over the hybrid cache -> (out [B,Hq,D], lse [B,Hq])."""
    qq = _u16(q)
    B, Hq, D = qq.shape
    c = {n: np.ascontiguousarray(cache[n]) for n in
         ("k_codes", "v_codes", "k_sz", "v_sz", "k_hi", "v_hi")}
    out = np.zeros((B, Hq, D), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    rc = _load().hqo_decode_attn(
        _p(qq), _p(c["k_codes"]), _p(c["v_codes"]), _p(bits(c["k_sz"])), _p(bits(c["v_sz"])),
        _p(bits(c["k_hi"])), _p(bits(c["v_hi"])), B, Hq, Hkv, D, int(cache["n_lo"]),
        int(cache["n_hi"]), int(cache["bits"]), int(cache["group"]), int(cache.get("fmt", FMT_INT)),
        default_scale(D) if scale is None else scale, _p(out), _p(lse))
    assert rc == 0, rc
    return out, lse


def prefill_quant(q, k, idx, kblock: int = 64, fmt: int = FMT_INT):
    """INT8 (fmt 0) or E4M3 (fmt 1, bits in the int8 arrays) codes + fp32
    scales.  Q per token: qi8 [B,Hq,N,D], sq [B,Hq,N].  K over the remaining
    (non-vertical) keys in position order, one scale per kblock of them:
    ki8 [B,Hkv,N-kv,D], sk [B,Hkv,ceil((N-kv)/kblock)]."""
    qq, kk = _u16(q), _u16(k)
    B, Hq, N, D = qq.shape
    Hkv = kk.shape[1]
    idx = np.ascontiguousarray(idx, np.int32)
    kv = idx.shape[2]
    nr = N - kv
    nblk = (nr + kblock - 1) // kblock
    qi8 = np.zeros((B, Hq, N, D), np.int8)
    sq = np.zeros((B, Hq, N), np.float32)
    ki8 = np.zeros((B, Hkv, nr, D), np.int8)
    sk = np.zeros((B, Hkv, nblk), np.float32)
    rc = _load().hqo_prefill_quant(_p(qq), _p(kk), _p(idx), B, Hq, Hkv, N, D, kv, kblock, fmt,
                                   _p(qi8), _p(sq), _p(ki8), _p(sk))
    assert rc == 0, rc
    return qi8, sq, ki8, sk


def prefill_attn(q, k, v, idx, window: int, quant=None, rows=None, kblock: int = 64,
                 scale: float | None = None, fmt: int = FMT_INT) -> np.ndarray:
    """Hybrid prefill attention, fp64 [B, Hq, nrows, D] for the given query rows."""
    qq, kk, vv = _u16(q), _u16(k), _u16(v)
    B, Hq, N, D = qq.shape
    Hkv = kk.shape[1]
    idx = np.ascontiguousarray(idx, np.int32)
    kv = idx.shape[2]
    if quant is None:
        quant = prefill_quant(qq, kk, idx, kblock, fmt)
    qi8, sq, ki8, sk = (np.ascontiguousarray(a) for a in quant)
    r = None if rows is None else np.ascontiguousarray(rows, np.int32)
    nrows = N if r is None else int(r.shape[0])
    out = np.zeros((B, Hq, nrows, D), np.float64)
    rc = _load().hqo_prefill_attn(_p(qq), _p(kk), _p(vv), _p(idx), _p(qi8), _p(sq), _p(ki8),
                                  _p(sk), B, Hq, Hkv, N, D, window, kv, kblock, fmt,
                                  default_scale(D) if scale is None else scale, _p(r), nrows,
                                  _p(out))
    assert rc == 0, rc
    return out
