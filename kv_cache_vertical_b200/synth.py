"""Seeded synthetic inputs for hybrid-precision attention.

This module only draws random tensors; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may be fed from it.

Recipe (per batch element b and KV head h_kv, each with its own PCG64
substream spawned from the workload seed, so the result does not depend on
threading):
  * u       -- a unit direction in R^D shared by that KV head's keys and the
               queries of its G query heads;
  * K       -- N(0, 1); 4 seeded "outlier" channels are multiplied by 10;
               then floor(f * L) seeded positions in [0, L - W) are
               overwritten with 3u + 0.3 N(0, 1) (planted vertical lines);
  * V       -- N(0, 1);
  * Q       -- N(0, 1) + 2u for every query row of every query head in the
               group (one row for decode, N rows for prefill);
  * probe   -- decode only: 64 extra prefix queries per query head, drawn like
               Q, sitting at positions L - 64 .. L - 1;
all rounded to bf16 (round to nearest even).  The shapes mimic Llama-3.1-8B /
70B-style GQA attention layers at long context (the pages evaluate
Llama-3.1-8B-Instruct, Qwen3 and GLM-4 models on LongBench-style long inputs;
these synthetic tensors stand in for those activations).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from fractions import Fraction

import numpy as np
import torch

PROBE_ROWS = 64
GROUP = 32


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str           # "decode" or "prefill"
    B: int
    Hq: int
    Hkv: int
    D: int
    L: int              # cached context (decode) or sequence length (prefill)
    window: int
    frac: Fraction      # vertical fraction f; k = floor(f * L)
    bits: int = 4       # KV code width for decode
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def k_vert(self) -> int:
        return (self.L * self.frac.numerator) // self.frac.denominator

    @property
    def n_lo(self) -> int:
        return self.L - self.window - self.k_vert

    @property
    def n_hi(self) -> int:
        return self.k_vert + self.window

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


F5 = Fraction(5, 100)
F25 = Fraction(25, 1000)

# The five workloads of the specification (sizes as stated there).
WORKLOADS = {
    "tiny_decode": Workload("tiny_decode", "decode", 1, 2, 1, 64, 1024, 128, F5, 4, 20260000),
    "llama8b_decode_32k": Workload("llama8b_decode_32k", "decode", 1, 32, 8, 128, 32768, 128,
                                   F5, 4, 20260001),
    "batched_decode_128k_int4": Workload("batched_decode_128k_int4", "decode", 8, 32, 8, 128,
                                         131072, 128, F5, 4, 20260002),
    "batched_decode_128k_int8": Workload("batched_decode_128k_int8", "decode", 8, 32, 8, 128,
                                         131072, 128, F5, 8, 20260002),
    "llama8b_prefill_32k": Workload("llama8b_prefill_32k", "prefill", 1, 32, 8, 128, 32768, 128,
                                    F5, 4, 20260003),
    "70b_decode_64k": Workload("70b_decode_64k", "decode", 32, 64, 8, 128, 65536, 256, F25, 4,
                               20260004),
}


def _substream(seed: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(b, h))))


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a).to(torch.bfloat16)


def make_inputs(w: Workload, threads: int | None = None, pin: bool = False) -> dict:
    """Draw the workload's tensors on the host (bf16, contiguous).

    decode:  q [B,Hq,D], q_probe [B,Hq,64,D], k, v [B,Hkv,L,D]
    prefill: q [B,Hq,N,D], k, v [B,Hkv,N,D]
    plus planted [B,Hkv,k] (the seeded vertical positions; for information).
    """
    B, Hq, Hkv, D, L, G = w.B, w.Hq, w.Hkv, w.D, w.L, w.G
    kv = w.k_vert
    nq = 1 if w.mode == "decode" else L

    def alloc(*shape):
        t = torch.empty(shape, dtype=torch.bfloat16)
        return t.pin_memory() if pin else t

    k = alloc(B, Hkv, L, D)
    v = alloc(B, Hkv, L, D)
    q = alloc(B, Hq, nq, D)
    qp = alloc(B, Hq, PROBE_ROWS, D) if w.mode == "decode" else None
    planted = torch.empty(B, Hkv, kv, dtype=torch.int32)

    def one(bh):
        b, h = divmod(bh, Hkv)
        rng = _substream(w.seed, b, h)
        u = rng.standard_normal(D)
        u = (u / np.linalg.norm(u)).astype(np.float32)
        outl = rng.choice(D, 4, replace=False)
        pos = np.sort(rng.choice(L - w.window, kv, replace=False)) if kv else np.zeros(0, np.int64)
        kk = rng.standard_normal((L, D), dtype=np.float32)
        kk[:, outl] *= 10.0
        kk[pos] = 3.0 * u + 0.3 * rng.standard_normal((kv, D), dtype=np.float32)
        k[b, h].copy_(_bf16(kk))
        v[b, h].copy_(_bf16(rng.standard_normal((L, D), dtype=np.float32)))
        for g in range(G):
            qq = rng.standard_normal((nq, D), dtype=np.float32) + 2.0 * u
            q[b, h * G + g].copy_(_bf16(qq))
            if qp is not None:
                pr = rng.standard_normal((PROBE_ROWS, D), dtype=np.float32) + 2.0 * u
                qp[b, h * G + g].copy_(_bf16(pr))
        planted[b, h] = torch.from_numpy(pos.astype(np.int32))

    n = B * Hkv
    threads = threads or min(n, os.cpu_count() or 1, 32)
    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(n)))
    else:
        for bh in range(n):
            one(bh)
    out = dict(k=k, v=v, planted=planted)
    if w.mode == "decode":
        out.update(q=q.view(B, Hq, D), q_probe=qp)
    else:
        out.update(q=q)
    return out


def make_inputs_device(w: Workload, device, seed_offset: int = 0) -> dict:
    """The recipe of make_inputs drawn directly on the GPU with torch's seeded
    generator (a different stream of numbers than the host generator's, the
    same distributions and structure).  For timing runs at full size, where
    drawing gigabytes on the host would take minutes; parity tests use
    make_inputs.  Decode workloads only (q [B,Hq,D], q_probe [B,Hq,64,D])."""
    assert w.mode == "decode"
    B, Hq, Hkv, D, L, G, W = w.B, w.Hq, w.Hkv, w.D, w.L, w.G, w.window
    kv = w.k_vert
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + seed_offset)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    u = torch.randn(B, Hkv, D, **f32)
    u /= u.norm(dim=-1, keepdim=True)
    k = torch.empty(B, Hkv, L, D, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    planted = torch.empty(B, Hkv, kv, dtype=torch.int32, device=device)
    for b in range(B):                       # one batch element at a time bounds the fp32 temporaries
        kk = torch.randn(Hkv, L, D, **f32)
        outl = torch.rand(Hkv, D, **f32).argsort(dim=-1)[:, :4]
        mult = torch.ones(Hkv, D, device=device).scatter_(1, outl, 10.0)
        kk *= mult[:, None, :]
        if kv:
            pos = torch.rand(Hkv, L - W, **f32).argsort(dim=-1)[:, :kv].sort(dim=-1).values
            rows = 3.0 * u[b][:, None, :] + 0.3 * torch.randn(Hkv, kv, D, **f32)
            kk.scatter_(1, pos[..., None].expand(-1, -1, D), rows)
            planted[b] = pos.to(torch.int32)
        k[b] = kk.to(torch.bfloat16)
        del kk
        v[b] = torch.randn(Hkv, L, D, **f32).to(torch.bfloat16)
    q = (torch.randn(B, Hkv, G, D, **f32) + 2.0 * u[:, :, None, :]).to(torch.bfloat16)
    qp = (torch.randn(B, Hkv, G, PROBE_ROWS, D, **f32) + 2.0 * u[:, :, None, None, :]).to(torch.bfloat16)
    return dict(k=k, v=v, planted=planted, q=q.view(B, Hq, D), q_probe=qp.view(B, Hq, PROBE_ROWS, D))
