"""ctypes binding of libhq.so (include/hq.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libhq.so.  PyTorch supplies device memory and the current CUDA
stream.  The ``hq_*`` functions mirror the C entry points one to one (device
tensors in, status checked); the lower-case helpers allocate outputs and
workspaces with torch and then call them.

There is no CPU fallback: importing this module raises if libhq.so is
missing, and every call needs CUDA tensors.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m kv_cache_vertical_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

HQ_OK = 0
HQ_DEV_BAD_INDEX = 0x1
HQ_DEV_TIMEOUT = 0x2
HQ_KV_INT, HQ_KV_FP8 = 0, 1      # low-bit code formats (hq_kv_cache.fmt)


class hq_kv_cache(ctypes.Structure):
    _fields_ = [("k_codes", _P), ("v_codes", _P), ("k_sz", _P), ("v_sz", _P), ("k_hi", _P),
                ("v_hi", _P), ("lo_pos", _P), ("n_lo", _I), ("n_hi", _I), ("bits", _I),
                ("group", _I), ("lo_cap", _I), ("fmt", _I)]


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_status_string = _sig("hq_status_string", ctypes.c_char_p, _I)
hq_version = _sig("hq_version", _I)
_read_status = _sig("hq_read_device_status", _I, _P, _I, ctypes.POINTER(ctypes.c_uint32), _P)
hq_probe_workspace_size = _sig("hq_probe_workspace_size", _SZ, _I, _I, _I, _I, _I, _I)
_probe = _sig("hq_probe_vertical", _I, _P, ctypes.c_int64, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
              _P, _P, _P, _SZ, _P)
hq_probe_shard_workspace_size = _sig("hq_probe_shard_workspace_size", _SZ, _I, _I, _I, _I, _I, _I, _I)
_pshard_stats = _sig("hq_probe_shard_stats", _I, _P, ctypes.c_int64, _P, _I, _I, _I, _I, _I, _I, _I,
                     _I, _F, _P, _P, _SZ, _P)
_pmerge_stats = _sig("hq_probe_merge_stats", _I, _P, _I, _I, _P, _P)
_pshard_topk = _sig("hq_probe_shard_topk", _I, _P, ctypes.c_int64, _P, _I, _I, _I, _I, _I, _I, _I,
                    _I, _I, _I, _F, _P, _P, _P, _P, _SZ, _P)
hq_probe_merge_workspace_size = _sig("hq_probe_merge_workspace_size", _SZ, _I, _I, _I, _I)
_pmerge_topk = _sig("hq_probe_merge_topk", _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P)
_pack = _sig("hq_pack_kv", _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
             ctypes.POINTER(hq_kv_cache), _P, _SZ, _P)
hq_decode_workspace_size = _sig("hq_decode_workspace_size", _SZ, _I, _I, _I, _I, _I, _I, _I)
_decode = _sig("hq_decode_attn", _I, _P, ctypes.POINTER(hq_kv_cache), _I, _I, _I, _I, _F, _P, _P,
               _P, _SZ, _P)
_append = _sig("hq_kv_append", _I, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.POINTER(hq_kv_cache), _P)
_pack_part = _sig("hq_pack_kv_part", _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                  ctypes.POINTER(hq_kv_cache), _P, _SZ, _P)
_append_part = _sig("hq_kv_append_part", _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                    ctypes.POINTER(hq_kv_cache), _P)
_merge = _sig("hq_decode_merge", _I, _P, _P, _I, _I, _I, _I, _P, _P, _P)
_decode_static = _sig("hq_decode_attn_static", _I, _P, ctypes.POINTER(hq_kv_cache), _I, _I, _I,
                      _I, _F, _P, _P, _P)
_read_static_status = _sig("hq_read_static_status", _I, _I, ctypes.POINTER(ctypes.c_uint32), _P)
_pquant = _sig("hq_prefill_quant", _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P)
hq_prefill_workspace_size = _sig("hq_prefill_workspace_size", _SZ, _I, _I, _I, _I, _I, _I)
_prefill = _sig("hq_prefill_attn", _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P,
                _SZ, _P)
_prefill_supported = _sig("hq_prefill_supported", _I, _I, _I, _I, _I)
_pquant_ex = _sig("hq_prefill_quant_ex", _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P)
_prefill_ex = _sig("hq_prefill_attn_ex", _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P,
                   _P, _SZ, _P)

EXPORTED = ["hq_status_string", "hq_version", "hq_read_device_status", "hq_probe_workspace_size",
            "hq_probe_vertical", "hq_pack_kv", "hq_decode_workspace_size", "hq_decode_attn",
            "hq_prefill_quant", "hq_prefill_workspace_size", "hq_prefill_attn",
            "hq_decode_attn_static", "hq_read_static_status", "hq_kv_append", "hq_decode_merge", "hq_prefill_quant_ex",
            "hq_prefill_attn_ex", "hq_probe_shard_workspace_size", "hq_probe_shard_stats",
            "hq_probe_merge_stats", "hq_probe_shard_topk", "hq_probe_merge_workspace_size",
            "hq_probe_merge_topk", "hq_prefill_supported", "hq_pack_kv_part",
            "hq_kv_append_part"]

HQ_ERR_SCRATCH_LIMIT = 7
STATIC_SCRATCH_BYTES = 16 << 20


class HQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {hq_status_string(status)}")


def hq_status_string(status: int) -> str:
    return _status_string(status).decode()


def _check(rc: int, what: str):
    if rc != HQ_OK:
        raise HQError(rc, what)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhq takes CUDA tensors only")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed device workspace (the library keeps it reusable afterwards)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def hq_read_device_status(ws: torch.Tensor, clear: bool = False, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(_read_status(_ptr(ws), int(clear), ctypes.byref(v), _stream(stream)),
           "hq_read_device_status")
    return v.value


# ---------------------------------------------------------------------------
# Hybrid KV cache
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class KVCache:
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_sz: torch.Tensor
    v_sz: torch.Tensor
    k_hi: torch.Tensor
    v_hi: torch.Tensor
    lo_pos: torch.Tensor | None
    n_lo: int
    n_hi: int
    bits: int
    group: int = 32
    fmt: int = HQ_KV_INT

    @classmethod
    def empty(cls, B, Hkv, L, D, window, k_vert, bits, device="cuda", with_pos=True,
              lo_cap=None, fmt=HQ_KV_INT):
        """Buffers for a cache of L tokens.  lo_cap (default: exactly the
        n_lo low rows) reserves low rows per (b, kv head) for decode appends."""
        return cls.alloc(B, Hkv, D, L - window - k_vert, k_vert + window, bits, device, with_pos,
                         lo_cap, fmt)

    @classmethod
    def alloc(cls, B, Hkv, D, n_lo, n_hi, bits, device="cuda", with_pos=True, lo_cap=None,
              fmt=HQ_KV_INT):
        """Buffers for n_lo low rows (lo_cap allocated) and n_hi bf16 rows."""
        C = n_lo if lo_cap is None else int(lo_cap)
        assert C >= n_lo, "lo_cap below the number of low rows"
        u8 = dict(dtype=torch.uint8, device=device)
        return cls(
            k_codes=torch.empty(B, Hkv, C, D * bits // 8, **u8),
            v_codes=torch.empty(B, Hkv, C, D * bits // 8, **u8),
            k_sz=torch.empty(B, Hkv, C, D // 32, 2, dtype=torch.float16, device=device),
            v_sz=torch.empty(B, Hkv, C, D // 32, 2, dtype=torch.float16, device=device),
            k_hi=torch.empty(B, Hkv, n_hi, D, dtype=torch.bfloat16, device=device),
            v_hi=torch.empty(B, Hkv, n_hi, D, dtype=torch.bfloat16, device=device),
            lo_pos=torch.empty(B, Hkv, C, dtype=torch.int32, device=device) if with_pos else None,
            n_lo=n_lo, n_hi=n_hi, bits=bits, fmt=fmt)

    @property
    def lo_cap(self) -> int:
        """Rows between consecutive (b, kv head) slices of the low arrays (the
        allocation, or the parent's for a row view)."""
        t = self.k_codes
        if t.dim() != 4:
            return self.n_lo
        return t.stride(1) // t.stride(2) if t.shape[2] > 0 else t.shape[2]

    def rows_part(self, lo_start: int, lo_end: int, hi_start: int = 0, hi_end: int = 0) -> "KVCache":
        """The cache restricted to low rows [lo_start, lo_end) (views, no copy:
        the low arrays keep their row stride through lo_cap) and bf16 rows
        [hi_start, hi_end) (copied unless that is every bf16 row, since the
        bf16 arrays carry no row stride).  Attention over the union of
        disjoint parts equals attention over the cache."""
        sl = slice(lo_start, lo_end)
        if (hi_start, hi_end) == (0, self.n_hi):
            k_hi, v_hi = self.k_hi, self.v_hi
        else:
            k_hi = self.k_hi[:, :, hi_start:hi_end].contiguous()
            v_hi = self.v_hi[:, :, hi_start:hi_end].contiguous()
        return KVCache(
            k_codes=self.k_codes[:, :, sl], v_codes=self.v_codes[:, :, sl],
            k_sz=self.k_sz[:, :, sl], v_sz=self.v_sz[:, :, sl], k_hi=k_hi, v_hi=v_hi,
            lo_pos=self.lo_pos[:, :, sl] if self.lo_pos is not None else None,
            n_lo=lo_end - lo_start, n_hi=hi_end - hi_start, bits=self.bits,
            group=self.group, fmt=self.fmt)

    def struct(self) -> hq_kv_cache:
        return hq_kv_cache(_ptr(self.k_codes), _ptr(self.v_codes), _ptr(self.k_sz),
                           _ptr(self.v_sz), _ptr(self.k_hi), _ptr(self.v_hi), _ptr(self.lo_pos),
                           self.n_lo, self.n_hi, self.bits, self.group,
                           self.lo_cap if self.n_lo > 0 else 0, self.fmt)

    def nbytes(self, with_pos: bool = False) -> int:
        """Bytes of the rows in use (spare low rows not counted)."""
        lo = [self.k_codes, self.v_codes, self.k_sz, self.v_sz]
        if with_pos and self.lo_pos is not None:
            lo.append(self.lo_pos)
        n = sum(t[:, :, :self.n_lo].numel() * t.element_size() for t in lo)
        return n + sum(t.numel() * t.element_size() for t in (self.k_hi, self.v_hi))


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def hq_probe_vertical(q_probe, q_head_stride, k, B, Hq, Hkv, P, L, D, window, k_vert,
                      softmax_scale, idx_out, score_out, ws, stream=None):
    _check(_probe(_ptr(q_probe), int(q_head_stride), _ptr(k), B, Hq, Hkv, P, L, D, window, k_vert,
                  float(softmax_scale), _ptr(idx_out), _ptr(score_out), _ptr(ws),
                  ws.numel() if ws is not None else 0, _stream(stream)), "hq_probe_vertical")


def hq_probe_shard_stats(q_probe, q_head_stride, k_shard, B, Hq, Hkv, P, Ls, D, key_off, L,
                         softmax_scale, stats_out, ws, stream=None):
    _check(_pshard_stats(_ptr(q_probe), int(q_head_stride), _ptr(k_shard), B, Hq, Hkv, P, Ls, D,
                         key_off, L, float(softmax_scale), _ptr(stats_out), _ptr(ws),
                         ws.numel() if ws is not None else 0, _stream(stream)), "hq_probe_shard_stats")


def hq_probe_merge_stats(parts, R, nrows, stats_out, stream=None):
    _check(_pmerge_stats(_ptr(parts), R, nrows, _ptr(stats_out), _stream(stream)),
           "hq_probe_merge_stats")


def hq_probe_shard_topk(q_probe, q_head_stride, k_shard, B, Hq, Hkv, P, Ls, D, key_off, L, window,
                        k_vert, softmax_scale, stats, cand_idx, cand_score, ws, stream=None):
    _check(_pshard_topk(_ptr(q_probe), int(q_head_stride), _ptr(k_shard), B, Hq, Hkv, P, Ls, D,
                        key_off, L, window, k_vert, float(softmax_scale), _ptr(stats), _ptr(cand_idx),
                        _ptr(cand_score), _ptr(ws), ws.numel() if ws is not None else 0,
                        _stream(stream)), "hq_probe_shard_topk")


def hq_probe_merge_topk(cand_idx, cand_score, R, B, Hkv, L, window, k_vert, idx_out, ws,
                        stream=None):
    _check(_pmerge_topk(_ptr(cand_idx), _ptr(cand_score), R, B, Hkv, L, window, k_vert,
                        _ptr(idx_out), _ptr(ws), ws.numel() if ws is not None else 0,
                        _stream(stream)), "hq_probe_merge_topk")


def hq_pack_kv(k, v, idx, B, Hkv, L, D, window, k_vert, bits, group, cache: KVCache, ws=None,
               stream=None):
    st = cache.struct()
    _check(_pack(_ptr(k), _ptr(v), _ptr(idx), B, Hkv, L, D, window, k_vert, bits, group,
                 ctypes.byref(st), _ptr(ws), ws.numel() if ws is not None else 0,
                 _stream(stream)), "hq_pack_kv")


def hq_pack_kv_part(k, v, idx, B, Hkv, L, D, window, k_vert, bits, group, lo0, hi0,
                    cache: KVCache, ws=None, stream=None):
    st = cache.struct()
    _check(_pack_part(_ptr(k), _ptr(v), _ptr(idx), B, Hkv, L, D, window, k_vert, bits, group, lo0,
                      hi0, ctypes.byref(st), _ptr(ws), ws.numel() if ws is not None else 0,
                      _stream(stream)), "hq_pack_kv_part")


def hq_kv_append_part(k_new, v_new, B, Hkv, D, L, window, k_vert, lo0, hi0, cache: KVCache,
                      stream=None):
    st = cache.struct()
    _check(_append_part(_ptr(k_new), _ptr(v_new), B, Hkv, D, L, window, k_vert, lo0, hi0,
                        ctypes.byref(st), _stream(stream)), "hq_kv_append_part")


def hq_kv_append(k_new, v_new, B, Hkv, D, L, window, k_vert, cache: KVCache, stream=None):
    st = cache.struct()
    _check(_append(_ptr(k_new), _ptr(v_new), B, Hkv, D, L, window, k_vert, ctypes.byref(st),
                   _stream(stream)), "hq_kv_append")


def hq_decode_merge(part_out, part_lse, R, B, Hq, D, out, lse_out, stream=None):
    _check(_merge(_ptr(part_out), _ptr(part_lse), R, B, Hq, D, _ptr(out), _ptr(lse_out),
                  _stream(stream)), "hq_decode_merge")


def hq_decode_attn(q, cache: KVCache, B, Hq, Hkv, D, softmax_scale, out, lse_out, ws, stream=None):
    st = cache.struct()
    _check(_decode(_ptr(q), ctypes.byref(st), B, Hq, Hkv, D, float(softmax_scale), _ptr(out),
                   _ptr(lse_out), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "hq_decode_attn")


def hq_decode_attn_static(q, cache: KVCache, B, Hq, Hkv, D, softmax_scale, out, lse_out,
                          stream=None):
    """Decode without a workspace argument: for callers that cannot allocate
    device memory when they call (stream capture in progress, memory fixed at
    start-up).  Its scratch is the library's fixed device array; make the first
    call on each device before any stream capture begins, and do not overlap
    calls on the GPU."""
    st = cache.struct()
    _check(_decode_static(_ptr(q), ctypes.byref(st), B, Hq, Hkv, D, float(softmax_scale),
                          _ptr(out), _ptr(lse_out), _stream(stream)), "hq_decode_attn_static")


def hq_read_static_status(clear: bool = False, stream=None) -> int:
    """Device status word of the last hq_decode_attn_static call on the
    current device (HQ_DEV_* bits; synchronizes the stream)."""
    v = ctypes.c_uint32(0)
    _check(_read_static_status(int(clear), ctypes.byref(v), _stream(stream)),
           "hq_read_static_status")
    return v.value


def hq_prefill_quant(q, k, idx, B, Hq, Hkv, N, D, k_vert, qi8, sq, ki8, sk, stream=None):
    _check(_pquant(_ptr(q), _ptr(k), _ptr(idx), B, Hq, Hkv, N, D, k_vert, _ptr(qi8), _ptr(sq),
                   _ptr(ki8), _ptr(sk), _stream(stream)), "hq_prefill_quant")


def hq_prefill_quant_ex(q, k, idx, B, Hq, Hkv, N, D, k_vert, low_fmt, qi8, sq, ki8, sk,
                        stream=None):
    _check(_pquant_ex(_ptr(q), _ptr(k), _ptr(idx), B, Hq, Hkv, N, D, k_vert, low_fmt, _ptr(qi8),
                      _ptr(sq), _ptr(ki8), _ptr(sk), _stream(stream)), "hq_prefill_quant_ex")


def hq_prefill_supported(D, Hq, Hkv, low_fmt=HQ_KV_INT) -> int:
    """HQ_OK (0) when a prefill of this shape and low-part format runs the
    tensor-core kernel on the current device, else HQ_ERR_UNSUPPORTED."""
    return _prefill_supported(D, Hq, Hkv, low_fmt)


def hq_prefill_attn_ex(q, k, v, idx, B, Hq, Hkv, N, D, window, k_vert, softmax_scale, low_fmt,
                       out, ws, stream=None):
    _check(_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, Hq, Hkv, N, D, window, k_vert,
                       float(softmax_scale), low_fmt, _ptr(out), _ptr(ws),
                       ws.numel() if ws is not None else 0, _stream(stream)), "hq_prefill_attn_ex")


def hq_prefill_attn(q, k, v, idx, B, Hq, Hkv, N, D, window, k_vert, softmax_scale, out, ws,
                    stream=None):
    _check(_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, Hq, Hkv, N, D, window, k_vert,
                    float(softmax_scale), _ptr(out), _ptr(ws), ws.numel() if ws is not None else 0,
                    _stream(stream)), "hq_prefill_attn")


# ---------------------------------------------------------------------------
# Convenience helpers (allocate with torch, then call the entry points)
# ---------------------------------------------------------------------------
def probe_vertical(q_probe, k, window, k_vert, scale=0.0, want_scores=False, ws=None):
    """q_probe: bf16 [B,Hq,P,D] (any head stride, rows contiguous); k: bf16 [B,Hkv,L,D]."""
    B, Hq, P, D = q_probe.shape
    Hkv, L = k.shape[1], k.shape[2]
    assert q_probe.stride(3) == 1 and q_probe.stride(2) == D and q_probe.stride(0) == Hq * q_probe.stride(1)
    idx = torch.empty(B, Hkv, k_vert, dtype=torch.int32, device=k.device)
    score = torch.empty(B, Hkv, L, dtype=torch.float32, device=k.device) if want_scores else None
    if ws is None:
        ws = workspace(hq_probe_workspace_size(B, Hq, Hkv, P, L, D), k.device)
    hq_probe_vertical(q_probe, q_probe.stride(1), k, B, Hq, Hkv, P, L, D, window, k_vert, scale,
                      idx, score, ws)
    return (idx, score) if want_scores else idx


def probe_context_plan(L: int, R: int):
    """Contiguous key ranges [key_off, key_off + Ls) of an L-key context for R
    ranks, as equal as possible (every rank gets at least one key when L >= R)."""
    return [(L * r // R, L * (r + 1) // R - L * r // R) for r in range(R)]


def probe_shard_stats(q_probe, k_shard, key_off, L, scale=0.0, ws=None):
    """Pass 1 on one rank's keys: (max, Z) per probe row, f32 [B, Hkv, G*P, 2]."""
    B, Hq, P, D = q_probe.shape
    Hkv, Ls = k_shard.shape[1], k_shard.shape[2]
    out = torch.empty(B, Hkv, (Hq // Hkv) * P, 2, dtype=torch.float32, device=k_shard.device)
    if ws is None:
        ws = workspace(hq_probe_shard_workspace_size(B, Hq, Hkv, P, Ls, D, 0), k_shard.device)
    hq_probe_shard_stats(q_probe, q_probe.stride(1), k_shard, B, Hq, Hkv, P, Ls, D, key_off, L,
                         scale, out, ws)
    return out


def probe_merge_stats(parts):
    """parts: f32 [R, B, Hkv, rows, 2] (max, Z) -> the context's (max, 1/Z)."""
    R = parts.shape[0]
    nrows = parts[0].numel() // 2
    out = torch.empty(parts.shape[1:], dtype=torch.float32, device=parts.device)
    hq_probe_merge_stats(parts.contiguous(), R, nrows, out)
    return out


def probe_shard_topk(q_probe, k_shard, key_off, L, window, k_vert, stats, scale=0.0, ws=None):
    """Pass 2 on one rank's keys with the context's row stats: the rank's best
    k_vert candidate columns (context positions, -1 padded) and their scores."""
    B, Hq, P, D = q_probe.shape
    Hkv, Ls = k_shard.shape[1], k_shard.shape[2]
    cand_idx = torch.empty(B, Hkv, k_vert, dtype=torch.int32, device=k_shard.device)
    cand_score = torch.empty(B, Hkv, k_vert, dtype=torch.float32, device=k_shard.device)
    if ws is None:
        ws = workspace(hq_probe_shard_workspace_size(B, Hq, Hkv, P, Ls, D, k_vert), k_shard.device)
    hq_probe_shard_topk(q_probe, q_probe.stride(1), k_shard, B, Hq, Hkv, P, Ls, D, key_off, L,
                        window, k_vert, scale, stats.contiguous(), cand_idx, cand_score, ws)
    return cand_idx, cand_score


def probe_merge_topk(cand_idx, cand_score, L, window, ws=None):
    """cand_idx / cand_score: [R, B, Hkv, k_vert] -> the context's index list."""
    R, B, Hkv, k_vert = cand_idx.shape
    idx = torch.empty(B, Hkv, k_vert, dtype=torch.int32, device=cand_idx.device)
    if ws is None:
        ws = workspace(hq_probe_merge_workspace_size(B, Hkv, L, window), cand_idx.device)
    hq_probe_merge_topk(cand_idx.contiguous(), cand_score.contiguous(), R, B, Hkv, L, window,
                        k_vert, idx, ws)
    return idx


def probe_context_parallel(q_probe, k_shard, key_off, L, window, k_vert, group=None, scale=0.0):
    """The vertical-column probe with the context's keys split over the ranks
    of `group` (torch.distributed): this rank holds keys [key_off, key_off +
    k_shard.shape[2]).  Two all-gathers (NCCL on device memory, gloo through
    the host): the probe rows' partial (max, Z), then every rank's top-k
    candidates.  Returns the context's index list on every rank."""
    B, Hq, P, D = q_probe.shape
    Hkv = k_shard.shape[1]
    empty = k_shard.shape[2] == 0          # more ranks than keys: this rank holds none
    if empty:
        st = torch.zeros(B, Hkv, (Hq // Hkv) * P, 2, dtype=torch.float32, device=q_probe.device)
        st[..., 0] = -torch.finfo(torch.float32).max
    else:
        st = probe_shard_stats(q_probe, k_shard, key_off, L, scale)
    stats = probe_merge_stats(torch.stack(_all_gather(st, group)))
    if empty:
        ci = torch.full((B, Hkv, k_vert), -1, dtype=torch.int32, device=q_probe.device)
        cs = torch.full((B, Hkv, k_vert), -torch.finfo(torch.float32).max, dtype=torch.float32,
                        device=q_probe.device)
    else:
        ci, cs = probe_shard_topk(q_probe, k_shard, key_off, L, window, k_vert, stats, scale)
    return probe_merge_topk(torch.stack(_all_gather(ci, group)), torch.stack(_all_gather(cs, group)),
                            L, window)


def pack_kv(k, v, idx, window, bits=4, ws=None, with_pos=True, lo_cap=None,
            fmt=HQ_KV_INT) -> KVCache:
    B, Hkv, L, D = k.shape
    k_vert = idx.shape[2]
    cache = KVCache.empty(B, Hkv, L, D, window, k_vert, bits, k.device, with_pos, lo_cap, fmt)
    hq_pack_kv(k, v, idx, B, Hkv, L, D, window, k_vert, bits, 32, cache, ws)
    return cache


def pack_kv_part(k, v, idx, window, part, bits=4, ws=None, with_pos=True, lo_cap=None,
                 fmt=HQ_KV_INT) -> KVCache:
    """One rank's part (lo0, lo1, hi0, hi1) of the cache pack_kv would build
    (a context split; see context_split_plan): only those rows are allocated
    and written, bit-identical to the whole cache's rows."""
    B, Hkv, L, D = k.shape
    k_vert = idx.shape[2]
    lo0, lo1, hi0, hi1 = part
    cache = KVCache.alloc(B, Hkv, D, lo1 - lo0, hi1 - hi0, bits, k.device, with_pos, lo_cap, fmt)
    hq_pack_kv_part(k, v, idx, B, Hkv, L, D, window, k_vert, bits, 32, lo0, hi0, cache, ws)
    return cache


def kv_append_part(part_cache: KVCache, part, k_new, v_new, L, window, k_vert, stream=None):
    """Token L enters a context-split cache on the rank whose part ends where
    the cache ends (the last rank of context_split_plan(..., window=W)); the
    other ranks' parts do not change.  The part's n_lo grows by one."""
    B, Hkv, D = k_new.shape
    lo0, _, hi0, _ = part
    hq_kv_append_part(k_new, v_new, B, Hkv, D, L, window, k_vert, lo0, hi0, part_cache, stream)
    part_cache.n_lo += 1
    return part_cache


def kv_append(cache: KVCache, k_new, v_new, L, window, stream=None):
    """Token L (bf16 [B, Hkv, D] key and value) enters the cache; the cache's
    n_lo grows by one (the position that left the window)."""
    B, Hkv, D = k_new.shape
    hq_kv_append(k_new, v_new, B, Hkv, D, L, window, cache.n_hi - window, cache, stream)
    cache.n_lo += 1
    return cache


def decode_attn(q, cache: KVCache, Hkv, scale=0.0, ws=None, want_lse=False):
    B, Hq, D = q.shape
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(hq_decode_workspace_size(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, cache.bits),
                       q.device)
    hq_decode_attn(q, cache, B, Hq, Hkv, D, scale, out, lse, ws)
    return (out, lse) if want_lse else out


def prefill_quant(q, k, idx, fmt=HQ_KV_INT):
    """Low-part pre-pass (INT8, or E4M3 code bits with fmt=HQ_KV_FP8): Q per
    row; K over the remaining (non-vertical) keys."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    k_vert = idx.shape[2]
    nr = N - k_vert
    nblk = (nr + 63) // 64
    qi8 = torch.empty(B, Hq, N, D, dtype=torch.int8, device=q.device)
    sq = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    ki8 = torch.empty(B, Hkv, nr, D, dtype=torch.int8, device=q.device)
    sk = torch.empty(B, Hkv, nblk, dtype=torch.float32, device=q.device)
    hq_prefill_quant_ex(q, k, idx, B, Hq, Hkv, N, D, k_vert, fmt, qi8, sq, ki8, sk)
    return qi8, sq, ki8, sk


def prefill_attn(q, k, v, idx, window, scale=0.0, ws=None, out=None, fmt=HQ_KV_INT):
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    k_vert = idx.shape[2]
    if out is None:
        out = torch.empty(B, Hq, N, D, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(hq_prefill_workspace_size(B, Hq, Hkv, N, D, k_vert), q.device)
    hq_prefill_attn_ex(q, k, v, idx, B, Hq, Hkv, N, D, window, k_vert, scale, fmt, out, ws)
    return out


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


# ---------------------------------------------------------------------------
# Context split of the decode across ranks
# ---------------------------------------------------------------------------
def context_split_plan(n_lo: int, n_hi: int, R: int, align: int = 64, window: int = 0):
    """Share the rows of one cache among R ranks for a context-split decode:
    rank r gets low rows [lo0, lo1) and bf16 rows [hi0, hi1).  Attention does
    not depend on the order of the rows, so any disjoint cover works; equal
    shares of both kinds give every rank the same bytes to read.  Low
    boundaries fall on multiples of `align` rows (whole decode tiles, 16-byte
    aligned views).  With window > 0 the last rank's bf16 rows include the
    whole window (the last `window` bf16 rows), so that decode appends
    (kv_append_part) touch that rank only.  Returns [(lo0, lo1, hi0, hi1)] * R."""
    if R < 1:
        raise ValueError("R must be at least 1")
    lo = [min(n_lo, (n_lo * r // R) // align * align) for r in range(R)] + [n_lo]
    hi = [n_hi * r // R for r in range(R + 1)]
    if window > 0:
        cap = max(0, n_hi - window)
        hi = [min(h, cap) for h in hi[:-1]] + [n_hi]
    return [(lo[r], lo[r + 1], hi[r], hi[r + 1]) for r in range(R)]


def _all_gather(t: torch.Tensor, group=None):
    """All-gather of a device tensor: NCCL gathers device memory directly;
    a process group without device collectives (gloo) gathers host copies."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        parts = [torch.empty_like(t) for _ in range(R)]
        dist.all_gather(parts, t, group=group)
        return parts
    th = t.cpu()
    parts = [torch.empty_like(th) for _ in range(R)]
    dist.all_gather(parts, th, group=group)
    return [x.to(t.device) for x in parts]


def decode_merge(part_out, part_lse):
    """Merge R partial decodes: part_out f32 [R, B, Hq, D], part_lse f32 [R, B, Hq]."""
    R, B, Hq, D = part_out.shape
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=part_out.device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=part_out.device)
    hq_decode_merge(part_out.contiguous(), part_lse.contiguous(), R, B, Hq, D, out, lse)
    return out, lse


def decode_context_parallel(q, part: KVCache, Hkv, group=None, scale=0.0):
    """Decode one step of a cache whose rows are split over the ranks of
    `group` (torch.distributed): `part` is this rank's rows (pack_kv_part with
    this rank's entry of context_split_plan, or rows_part of a replica).  Each
    rank decodes its part with its log-sum-exp, the (out, lse) pairs are
    all-gathered (NCCL on device memory, gloo through the host), and every
    rank merges them exactly.  Returns (out, lse) of the whole cache."""
    B, Hq, D = q.shape
    if part.n_lo + part.n_hi > 0:
        out_r, lse_r = decode_attn(q, part, Hkv, scale=scale, want_lse=True)
    else:
        out_r = torch.zeros(B, Hq, D, dtype=torch.float32, device=q.device)
        lse_r = torch.full((B, Hq), float("-inf"), dtype=torch.float32, device=q.device)
    outs = _all_gather(out_r, group)
    lses = _all_gather(lse_r, group)
    return decode_merge(torch.stack(outs), torch.stack(lses))
