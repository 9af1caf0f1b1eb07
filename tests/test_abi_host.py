"""Host-side checks of the C ABI: the library loads, exports every symbol gdn.h declares,
and rejects bad arguments before any launch (these calls never touch a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

import gated_deltanet_05_b200 as gdn
from gated_deltanet_05_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gdn_build.build()
    return gdn.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_functions()
    assert set(names) == set(gdn.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn_[a-z_]+)\b", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_status_strings_and_version(L):
    for code, name in gdn.STATUS.items():
        assert L.gdn_status_string(code).decode() == name
    assert L.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert L.gdn_version() == 100
    # only the tensor-core path (d_k = d_v = 128, chunk 64) uses scratch: one K ring
    # per SM id (none without a device)
    assert L.gdn_chunk_fwd_workspace_bytes(4, 16384, 16, 64, 64, 64) == 0
    assert L.gdn_chunk_fwd_workspace_bytes(4, 16384, 16, 128, 128, 32) == 0
    assert L.gdn_chunk_fwd_workspace_bytes(4, 16384, 16, 128, 128, 64) % (4 * 16384) == 0


def _cu(vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced on these paths


def _chunk(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, la=FAKE, b=FAKE, S0=None, cud=FAKE, cuh=_cu([0, 64]),
             n_seq=1, H=2, dk=128, dv=128, C=64, scale=1.0, y=FAKE, ydt=0, ST=None, ws=None,
             wsb=0, st=None)
    a.update(kw)
    return L.gdn_chunk_fwd(a["q"], a["k"], a["v"], a["dt"], a["la"], a["b"], a["S0"], a["cud"],
                           ctypes.cast(a["cuh"], ctypes.c_void_p) if a["cuh"] is not None else None,
                           a["n_seq"], a["H"], a["dk"], a["dv"], a["C"], a["scale"], a["y"],
                           a["ydt"], a["ST"], a["ws"], a["wsb"], a["st"])


def test_chunk_fwd_rejects_bad_arguments(L):
    assert _chunk(L, cuh=None) == 1                         # no host cu_seqlens
    assert _chunk(L, n_seq=-1) == 1
    assert _chunk(L, H=0) == 1
    assert _chunk(L, dt=7) == 1                             # unknown dtype
    assert _chunk(L, ydt=3) == 1
    assert _chunk(L, dk=96) == 2                            # unsupported sizes
    assert _chunk(L, dv=256) == 2
    assert _chunk(L, C=128) == 2
    assert _chunk(L, C=8) == 2
    assert _chunk(L, cuh=_cu([1, 64])) == 1                 # must start at 0
    assert _chunk(L, cuh=_cu([0, 64, 32]), n_seq=2) == 1    # must not decrease
    assert _chunk(L, q=None) == 1                           # null input
    assert _chunk(L, y=ctypes.c_void_p(0x10008)) == 1       # misaligned output
    assert _chunk(L, la=ctypes.c_void_p(0x10002)) == 1      # misaligned gate
    assert _chunk(L, n_seq=0, cuh=_cu([0])) == 0            # nothing to do
    assert _chunk(L) != 0                                   # tensor-core path without its workspace


def test_selftest_rejects_bad_arguments(L):
    assert L.gdn_selftest_bounded_wait(0, 0, None) == 1          # limit out of range
    assert L.gdn_selftest_bounded_wait(3_000_000_000, 0, None) == 1
    assert L.gdn_selftest_bounded_wait(1000, 3, None) == 1       # unknown mode
    assert L.gdn_selftest_bounded_wait(1000, 1, None) == 1       # abort needs a long limit


def test_decode_and_gate_norm_reject_bad_arguments(L):
    dec = lambda **kw: L.gdn_decode_step(kw.get("q", FAKE), FAKE, FAKE, kw.get("dt", 0), FAKE,
                                         FAKE, kw.get("S", FAKE), kw.get("n", 4), kw.get("H", 2),
                                         kw.get("dk", 128), kw.get("dv", 128), 1.0, FAKE,
                                         kw.get("ydt", 0), None)
    assert dec(n=-1) == 1
    assert dec(ydt=2) == 1
    assert dec(dt=2) == 1
    assert dec(H=0) == 1
    assert dec(dk=48) == 2
    assert dec(dv=512) == 2
    assert dec(q=None) == 1
    assert dec(S=ctypes.c_void_p(0x10004)) == 1
    assert dec(n=0) == 0
    gn = lambda **kw: L.gdn_gate_norm(kw.get("y", FAKE), kw.get("dt", 1), FAKE, 1, FAKE,
                                      kw.get("rows", 10), kw.get("dv", 128), 1e-6,
                                      kw.get("o", FAKE), kw.get("odt", 1), None)
    assert gn(rows=-1) == 1
    assert gn(dv=96) == 2
    assert gn(dv=512) == 2
    assert gn(dt=5) == 1
    assert gn(odt=2) == 1
    assert gn(y=None) == 1
    assert gn(o=ctypes.c_void_p(0x10008)) == 1
    assert gn(rows=0) == 0


def test_backward_rejects_bad_arguments(L):
    cu = (ctypes.c_int32 * 3)(0, 64, 100)
    # per (chain, 64-token chunk): two 128 x 128 states, U~ and dU~ (64 x 128 each), the
    # chunk's cache (3 x 64 x 64 + 64 x 128 floats), and two 64-column value slices' blocks of
    # per-chunk sums (2 x 64 x 64 + 3 x 64 x 128 + 64 + 1 floats each)
    part = (64 * (2 * 64 + 3 * 128 + 1) + 1 + 3) // 4 * 4      # rounded up to a multiple of 4
    assert L.gdn_backward_workspace_bytes(ctypes.cast(cu, ctypes.c_void_p), 2, 2, 128, 128) == \
        2 * 2 * 1 * (2 * 128 * 128 + 2 * 64 * 128 + 64 * (3 * 64 + 128) + 2 * part) * 4
    assert L.gdn_backward_workspace_bytes(None, 2, 2, 128, 128) == 0

    def bw(**kw):
        c = kw.get("cu", cu)
        return L.gdn_backward(FAKE, FAKE, FAKE, kw.get("dt", 0), FAKE, FAKE, None, FAKE,
                              ctypes.cast(c, ctypes.c_void_p) if c is not None else None,
                              kw.get("n_seq", 2), kw.get("H", 2), kw.get("dk", 128), kw.get("dv", 128),
                              1.0, kw.get("dy", FAKE), None, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                              kw.get("ws", FAKE), kw.get("wsb", 1 << 30), None)
    assert bw(dt=2) == 1
    assert bw(dk=24) == 2
    assert bw(H=0) == 1
    assert bw(cu=None) == 1
    assert bw(cu=(ctypes.c_int32 * 3)(0, 64, 10)) == 1
    assert bw(dy=None) == 1
    assert bw(dy=ctypes.c_void_p(0x10008)) == 1     # dy must be 16-byte aligned
    assert bw(wsb=1000) == 1
    assert bw(ws=None) == 1
    assert bw(n_seq=0) == 0


def test_gate_norm_buffer_overlap(L):
    """o may be y itself with y's dtype (in place); any other overlap of o with y or z is
    rejected before a launch. 10 rows of d_v = 128: 2,560 bytes in bf16, 5,120 in fp32."""
    Y, Z = 0x100000, 0x200000
    p = ctypes.c_void_p
    gn = lambda y, ydt, z, o, odt: L.gdn_gate_norm(p(y), ydt, p(z), 1, FAKE, 10, 128, 1e-6, p(o), odt, None)
    assert gn(Y, 1, Z, Y, 0) == 1                 # in place needs one dtype
    assert gn(Y, 1, Z, Y + 2544, 1) == 1          # o starts inside y
    assert gn(Y + 2544, 1, Z, Y, 1) == 1          # y starts inside o
    assert gn(Y, 0, Z, Y + 4096, 1) == 1          # fp32 y reaches into o
    assert gn(Y, 1, Z, Z + 16, 1) == 1            # o overlaps z
    assert gn(Y, 1, Y, Y, 1) == 1                 # z is o


def test_chunk_fwd_gated_rejects_bad_arguments(L):
    cu = (ctypes.c_int32 * 3)(0, 64, 100)
    cu_bad = (ctypes.c_int32 * 3)(0, 64, 10)

    def g(**kw):
        c = kw.get("cu", cu)
        return L.gdn_chunk_fwd_gated(FAKE, FAKE, FAKE, kw.get("dt", 1), FAKE, FAKE, None, FAKE,
                                     ctypes.cast(c, ctypes.c_void_p), kw.get("n_seq", 2), kw.get("H", 2),
                                     kw.get("dk", 128), kw.get("dv", 128), kw.get("chunk", 64), 1.0,
                                     kw.get("z", FAKE), kw.get("w", FAKE), kw.get("eps", 1e-6),
                                     kw.get("o", FAKE), kw.get("odt", 1), None, FAKE, 1 << 24, None)
    assert g(dt=0) == 2            # fp32 inputs: the one-call form covers the tensor-core path only
    assert g(dk=64) == 2
    assert g(chunk=32) == 2
    assert g(dt=4) == 1
    assert g(odt=3) == 1
    assert g(eps=-1.0) == 1
    assert g(H=0) == 1
    assert g(cu=cu_bad) == 1
    assert g(z=None) == 1
    assert g(w=None) == 1
    assert g(o=None) == 1
    assert g(o=ctypes.c_void_p(0x10008)) == 1
    assert g(z=ctypes.c_void_p(0x20000), o=ctypes.c_void_p(0x20010)) == 1   # o overlaps z
    assert g(n_seq=0) == 0


def test_decode_tokens_rejects_bad_arguments(L):
    dt = lambda **kw: L.gdn_decode_tokens(kw.get("q", FAKE), FAKE, FAKE, kw.get("dt", 0), FAKE, FAKE,
                                          kw.get("S", FAKE), kw.get("n", 4), kw.get("nt", 4),
                                          kw.get("H", 2), kw.get("dk", 128), kw.get("dv", 128), 1.0,
                                          FAKE, kw.get("ydt", 1), None)
    assert dt(nt=0) == 1
    assert dt(ydt=3) == 1
    assert dt(nt=9) == 1
    assert dt(n=-1) == 1
    assert dt(H=0) == 1
    assert dt(dt=2) == 1
    assert dt(dk=256) == 2
    assert dt(dv=24) == 2
    assert dt(q=None) == 1
    assert dt(S=ctypes.c_void_p(0x10004)) == 1
    assert dt(n=0) == 0


def test_featurize_rejects_bad_arguments(L):
    cu_ok = (ctypes.c_int32 * 3)(0, 5, 12)
    cu_bad = (ctypes.c_int32 * 3)(0, 7, 5)           # decreasing
    cu_short = (ctypes.c_int32 * 3)(0, 5, 11)        # does not reach n_tok

    def ft(**kw):
        cu = kw.get("cu", cu_ok)
        return L.gdn_featurize(kw.get("xq", FAKE), FAKE, FAKE, kw.get("dt", 1), FAKE, FAKE, FAKE,
                               kw.get("W", 4), FAKE, FAKE, FAKE, FAKE, FAKE,
                               ctypes.cast(cu, ctypes.c_void_p) if cu is not None else None,
                               kw.get("n_seq", 2), kw.get("n_tok", 12), kw.get("H", 2),
                               kw.get("dk", 128), kw.get("dv", 128), kw.get("eps", 1e-6),
                               kw.get("q", FAKE), FAKE, FAKE, FAKE, FAKE, None)
    assert ft(dt=3) == 1
    assert ft(W=0) == 1
    assert ft(W=5) == 1
    assert ft(H=0) == 1
    assert ft(n_seq=0) == 1
    assert ft(n_tok=-1) == 1
    assert ft(eps=-1.0) == 1
    assert ft(eps=float("nan")) == 1
    assert ft(dk=256) == 2
    assert ft(dv=48) == 2
    assert ft(cu=cu_bad) == 1
    assert ft(cu=cu_short) == 1
    assert ft(xq=None) == 1
    assert ft(q=None) == 1
    assert ft(q=ctypes.c_void_p(0x10008)) == 1     # not 16-byte aligned
    assert ft(n_tok=0, cu=(ctypes.c_int32 * 3)(0, 0, 0)) == 0


def test_binding_has_no_cpu_fallback(monkeypatch):
    """Calls on CPU tensors raise instead of computing anything."""
    import torch
    q = torch.zeros(4, 1, 16)
    with pytest.raises(ValueError):
        gdn.decode_step(q, q, q, torch.ones(4, 1), torch.ones(4, 1), torch.zeros(4, 1, 16, 16))
    with pytest.raises(ValueError):
        gdn.gate_norm(q, q, torch.zeros(16))


def test_package_does_not_import_oracle():
    pkg_dir = os.path.dirname(gdn.__file__)
    for root, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "gdn_oracle" not in text, f
