"""hq_decode_attn_static: decode whose scratch is the library's fixed device
array, for callers that cannot allocate device memory when they call (for
example while another component is capturing the stream into a CUDA graph, or
in a serving process whose device memory is fixed at start-up).

It must give what hq_decode_attn gives, call after call, although every call
reuses the same array.  This file is collected last on purpose, and it must
pass both on its own in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from hq_testutil import MAX_ABS, MEAN_ABS, to_dev
from kv_cache_vertical_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def hq():
    from kv_cache_vertical_b200 import hq as m
    return m


@pytest.mark.parametrize("name", ["llama8b_decode_32k", "tiny_decode", "batched_decode_128k_int8"])
def test_static_scratch_decode_matches_workspace_decode(name):
    H = hq()
    w = WORKLOADS[name]
    if name.startswith("batched"):
        w = w.replace(B=2, L=40000)          # INT8 codes, several (b, kv head) pairs
    x = make_inputs(w)
    d = to_dev(x)
    cache = H.pack_kv(d["k"], d["v"], d["planted"], w.window, w.bits)
    ref, ref_lse = H.decode_attn(d["q"], cache, w.Hkv, want_lse=True)
    for _ in range(2):                       # two calls in a row share the array
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        H.hq_decode_attn_static(d["q"], cache, w.B, w.Hq, w.Hkv, w.D, 0.0, out, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        err = (out.double() - ref.double()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, \
            f"max {err.max().item():.3e} mean {err.mean().item():.3e}"
        assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=1e-5)
        # the fixed array's status word: no bounded wait ran out, no bad input
        assert H.hq_read_static_status() == 0


def test_static_scratch_rejects_problems_beyond_its_size():
    H = hq()
    # Real (small) buffers, but dimensions whose split partials would need far
    # more than the fixed array: rejected on the host before anything launches.
    dev = "cuda"
    cache = H.KVCache(
        k_codes=torch.zeros(64, dtype=torch.uint8, device=dev),
        v_codes=torch.zeros(64, dtype=torch.uint8, device=dev),
        k_sz=torch.zeros(8, dtype=torch.float16, device=dev),
        v_sz=torch.zeros(8, dtype=torch.float16, device=dev),
        k_hi=torch.zeros(128, dtype=torch.bfloat16, device=dev),
        v_hi=torch.zeros(128, dtype=torch.bfloat16, device=dev),
        lo_pos=None, n_lo=100000, n_hi=1000, bits=4)
    B, Hq, Hkv, D = 4096, 64, 8, 128
    assert H.hq_decode_workspace_size(B, Hq, Hkv, D, cache.n_lo, cache.n_hi, 4) > H.STATIC_SCRATCH_BYTES
    q = torch.zeros(128, dtype=torch.bfloat16, device=dev)
    out = torch.zeros(128, dtype=torch.float32, device=dev)
    with pytest.raises(H.HQError) as e:
        H.hq_decode_attn_static(q, cache, B, Hq, Hkv, D, 0.0, out, None)
    assert e.value.status == H.HQ_ERR_SCRATCH_LIMIT


def test_static_scratch_covers_every_decode_workload():
    # The decode's scratch holds one partial slot per piece a CTA may write,
    # the pieces it may join included; its size depends on the device's SM
    # count and residency, so it is checked here, on the device.
    H = hq()
    for name, w in WORKLOADS.items():
        if w.mode != "decode":
            continue
        need = H.hq_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.n_lo, w.n_hi, w.bits)
        assert need <= H.STATIC_SCRATCH_BYTES, (name, need)
