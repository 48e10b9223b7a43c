"""Host-side tests of the C ABI (no GPU needed).

The library must load, export every entry point include/hq.h declares, and
reject bad arguments on the host before launching anything.  None of the calls
below reaches a kernel launch.
"""
import ctypes
import os
import re

import pytest

from kv_cache_vertical_b200 import build as hqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hq.h")


@pytest.fixture(scope="module")
def lib():
    path = hqbuild.build()
    return ctypes.CDLL(path)


def declared_symbols():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z_0-9]+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("hq_probe_vertical", "hq_pack_kv", "hq_decode_attn", "hq_prefill_attn",
              "hq_prefill_quant", "hq_status_string", "hq_read_device_status"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), f"libhq.so does not export {s}"


def test_binding_names_match_header():
    from kv_cache_vertical_b200 import hq
    assert sorted(hq.EXPORTED) == sorted(declared_symbols())


def test_status_strings(lib):
    lib.hq_status_string.restype = ctypes.c_char_p
    assert lib.hq_status_string(0) == b"HQ_OK"
    assert lib.hq_status_string(3) == b"HQ_ERR_WORKSPACE"
    assert lib.hq_status_string(99) == b"HQ_ERR_UNKNOWN"
    assert lib.hq_version() >= 100


class _Cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("k_codes", "v_codes", "k_sz", "v_sz", "k_hi", "v_hi", "lo_pos")] + \
               [(n, ctypes.c_int) for n in ("n_lo", "n_hi", "bits", "group", "lo_cap", "fmt")]


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced on the host
ODD = ctypes.c_void_p(0x10008)       # misaligned


def test_pack_argument_checks(lib):
    f = lib.hq_pack_kv
    f.restype = ctypes.c_int
    c = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1024 - 128 - 51, 51 + 128, 4, 32)
    args = lambda **kw: dict(dict(k=FAKE, v=FAKE, idx=FAKE, B=1, Hkv=1, L=1024, D=64, W=128,
                                  kv=51, bits=4, group=32), **kw)

    def call(**kw):
        a = args(**kw)
        return f(a["k"], a["v"], a["idx"], a["B"], a["Hkv"], a["L"], a["D"], a["W"], a["kv"],
                 a["bits"], a["group"], ctypes.byref(kw.get("cache", c)), None, ctypes.c_size_t(0),
                 None)
    assert call(k=None) == 1
    assert call(D=96) == 2
    assert call(bits=3) == 2
    assert call(group=64) == 2
    assert call(kv=1024 - 127) == 1          # k_vert > L - window
    assert call(L=1000) == 1                  # n_lo / n_hi inconsistent with the cache
    assert call(k=ODD) == 1                   # misaligned
    bad = _Cache(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, 845, 179, 4, 32)
    assert call(cache=bad) == 1               # missing hi buffer


def test_cache_struct_matches_header():
    """The binding's struct has the header's fields, in the header's order."""
    from kv_cache_vertical_b200 import hq
    text = open(os.path.join(ROOT, "include", "hq.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\} hq_kv_cache;", text).group(1)
    names = re.findall(r"(\w+);", body)
    assert names == [n for n, _ in hq.hq_kv_cache._fields_]
    assert [n for n, _ in _Cache._fields_] == names


def test_append_argument_checks(lib):
    f = lib.hq_kv_append
    f.restype = ctypes.c_int
    L, W, kv = 1024, 128, 51
    c = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, L - W - kv, kv + W, 4, 32, L - W - kv + 8)

    def call(k=FAKE, v=FAKE, B=1, Hkv=1, D=64, L=L, W=W, kv=kv, cache=c):
        return f(k, v, B, Hkv, D, L, W, kv, ctypes.byref(cache), None)
    assert call(k=None) == 1
    assert call(D=96) == 2
    assert call(L=L + 1) == 1                 # n_lo != L - window - k_vert
    assert call(W=W - 1, L=L - 1) == 1        # n_hi != k_vert + window
    assert call(v=ODD) == 1                   # misaligned
    full = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, L - W - kv, kv + W, 4, 32, L - W - kv)
    assert call(cache=full) == 1              # no spare low row
    exact = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, L - W - kv, kv + W, 4, 32, 0)
    assert call(cache=exact) == 1             # lo_cap 0 means exactly n_lo rows: no room
    small = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 845, 179, 4, 32, 800)
    lib.hq_decode_attn.restype = ctypes.c_int
    assert lib.hq_decode_attn(FAKE, ctypes.byref(small), 1, 2, 1, 64, ctypes.c_float(0.0), FAKE,
                              None, FAKE, ctypes.c_size_t(1 << 30), None) == 1   # lo_cap < n_lo


def test_decode_argument_checks(lib):
    f = lib.hq_decode_attn
    f.restype = ctypes.c_int
    lib.hq_decode_workspace_size.restype = ctypes.c_size_t
    c = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 845, 179, 4, 32)
    need = lib.hq_decode_workspace_size(1, 2, 1, 64, 845, 179, 4)
    assert need > 256

    def call(q=FAKE, cache=c, Hq=2, Hkv=1, D=64, out=FAKE, ws=FAKE, wsb=need):
        return f(q, ctypes.byref(cache), 1, Hq, Hkv, D, ctypes.c_float(0.0), out, None, ws,
                 ctypes.c_size_t(wsb), None)
    assert call(q=None) == 1
    assert call(out=None) == 1
    assert call(Hq=3, Hkv=2) == 1             # Hq % Hkv != 0
    assert call(Hq=12, Hkv=4) == 2            # G = 3 not supported
    assert call(D=80) == 2
    assert call(ws=None) == 3
    assert call(wsb=need - 1) == 3
    assert call(out=ODD) == 1
    bad = _Cache(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 845, 179, 5, 32)
    assert call(cache=bad) == 2
    assert lib.hq_decode_workspace_size(1, 2, 1, 96, 845, 179, 4) == 0


def test_probe_and_prefill_argument_checks(lib):
    p = lib.hq_probe_vertical
    p.restype = ctypes.c_int
    lib.hq_probe_workspace_size.restype = ctypes.c_size_t
    need = lib.hq_probe_workspace_size(1, 2, 1, 64, 1024, 64)

    def probe(P=64, L=1024, D=64, W=128, kv=51, stride=64 * 64, ws=FAKE, wsb=need, idx=FAKE):
        return p(FAKE, ctypes.c_int64(stride), FAKE, 1, 2, 1, P, L, D, W, kv, ctypes.c_float(0),
                 idx, None, ws, ctypes.c_size_t(wsb), None)
    assert probe(idx=None) == 1
    assert probe(P=2000) == 1                 # P > L
    assert probe(kv=1024 - 100) == 1          # k_vert > L - window
    assert probe(stride=100) == 1             # head stride smaller than P * D
    assert probe(D=32) == 2
    assert probe(ws=None) == 3
    assert probe(wsb=need - 1) == 3
    q = lib.hq_prefill_attn
    q.restype = ctypes.c_int
    lib.hq_prefill_workspace_size.restype = ctypes.c_size_t
    need = lib.hq_prefill_workspace_size(1, 4, 2, 256, 128, 12)

    def pre(N=256, D=128, Hq=4, Hkv=2, W=32, kv=12, idx=FAKE, ws=FAKE, wsb=need):
        return q(FAKE, FAKE, FAKE, idx, 1, Hq, Hkv, N, D, W, kv, ctypes.c_float(0), FAKE, ws,
                 ctypes.c_size_t(wsb), None)
    assert pre(idx=None) == 1
    assert pre(kv=300) == 1
    assert pre(D=256) == 2
    # the prefill attention has one kernel: head_dim 128, two query heads per CTA
    assert pre(D=64) == 2
    assert pre(Hq=2, Hkv=2) == 2
    assert pre(ws=None) == 3
    assert pre(wsb=need - 1) == 3
    sup = lib.hq_prefill_supported
    sup.restype = ctypes.c_int
    assert sup(64, 4, 2, 0) == 2 and sup(128, 2, 2, 0) == 2 and sup(128, 4, 2, 7) == 2
    qq = lib.hq_prefill_quant
    qq.restype = ctypes.c_int
    assert qq(FAKE, FAKE, FAKE, 1, 4, 2, 256, 64, 12, None, FAKE, FAKE, FAKE, None) == 1
    assert qq(FAKE, FAKE, None, 1, 4, 2, 256, 64, 12, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert qq(FAKE, FAKE, FAKE, 1, 4, 2, 256, 64, 300, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_build_module_imports_without_the_library():
    # `from kv_cache_vertical_b200 import build` is what builds libhq.so, so it
    # must not load the binding (which raises when the library is missing)
    import os
    import subprocess
    import sys
    code = ("import sys; from kv_cache_vertical_b200 import build; "
            "assert 'kv_cache_vertical_b200.hq' not in sys.modules, 'binding loaded'")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_prefill_format_argument_checks(lib):
    # the low-part format is checked on the host, before any launch: an
    # unknown format, and FP8 where the tensor-core kernel does not apply
    # (D = 64, or an odd number of query heads per KV head; on a machine
    # without a GPU the tensor-core kernel is never available)
    q = lib.hq_prefill_quant_ex
    q.restype = ctypes.c_int
    assert q(FAKE, FAKE, FAKE, 1, 2, 1, 256, 64, 8, 7, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert q(None, FAKE, FAKE, 1, 2, 1, 256, 64, 8, 1, FAKE, FAKE, FAKE, FAKE, None) == 1
    f = lib.hq_prefill_attn_ex
    f.restype = ctypes.c_int

    def call(D=128, Hq=2, Hkv=1, fmt=1, q=FAKE):
        return f(q, FAKE, FAKE, FAKE, 1, Hq, Hkv, 256, D, 32, 8, ctypes.c_float(0.0), fmt, FAKE,
                 FAKE, ctypes.c_size_t(1 << 30), None)
    assert call(fmt=7) == 2
    assert call(D=64, fmt=1) == 2
    assert call(Hq=3, Hkv=1, fmt=1) == 2
    assert call(q=None) == 1


def test_probe_split_argument_checks(lib):
    # host checks of the context-split probe, before any launch
    st = lib.hq_probe_shard_stats
    st.restype = ctypes.c_int

    def stats(Ls=100, key_off=0, L=300, P=64, q=FAKE, out=FAKE):
        return st(q, ctypes.c_int64(64 * 128), FAKE, 1, 2, 1, P, Ls, 128, key_off, L,
                  ctypes.c_float(0.0), out, FAKE, ctypes.c_size_t(1 << 30), None)
    assert stats(q=None) == 1
    assert stats(out=None) == 1
    assert stats(key_off=250) == 1            # key range past the context
    assert stats(Ls=0) == 1
    assert stats(P=301) == 1                  # more probe rows than context
    tk = lib.hq_probe_shard_topk
    tk.restype = ctypes.c_int

    def topk(k_vert=10, window=64, cand=FAKE):
        return tk(FAKE, ctypes.c_int64(64 * 128), FAKE, 1, 2, 1, 64, 100, 128, 0, 300, window,
                  k_vert, ctypes.c_float(0.0), FAKE, cand, FAKE, FAKE, ctypes.c_size_t(1 << 30), None)
    assert topk(k_vert=237) == 1              # k_vert > L - window
    assert topk(cand=None) == 1
    mg = lib.hq_probe_merge_topk
    mg.restype = ctypes.c_int
    assert mg(FAKE, FAKE, 0, 1, 1, 300, 64, 10, FAKE, FAKE, ctypes.c_size_t(1 << 30), None) == 1
    assert mg(FAKE, FAKE, 2, 1, 1, 300, 64, 10, FAKE, None, ctypes.c_size_t(0), None) == 3
    assert mg(None, None, 2, 1, 1, 300, 64, 0, None, None, ctypes.c_size_t(0), None) == 0
    ms = lib.hq_probe_merge_stats
    ms.restype = ctypes.c_int
    assert ms(FAKE, 0, 10, FAKE, None) == 1
