"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/swa.h declares, and rejects bad arguments on the host before any CUDA
call is made."""
import ctypes
import os
import re

import pytest

import decode_swa_prefill_b200 as swa
from decode_swa_prefill_b200 import build as swa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")


@pytest.fixture(scope="module")
def lib():
    swa_build.build()
    return swa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(swa_[a-z_]+)\s*\(", text)))


def test_header_and_exports_agree(lib):
    decl = declared_functions()
    assert decl == sorted(swa.EXPORTED)
    for name in decl:
        assert hasattr(lib, name), name


def test_exported_symbols_are_c_linkage():
    # nm -D lists the plain (unmangled) names
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", swa.library_path], capture_output=True,
                         text=True, check=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in names, name


def test_status_strings(lib):
    assert swa.swa_status_string(0) == "ok"
    assert swa.swa_status_string(4) == "device wait timed out"
    assert swa.swa_status_string(5) == "device consistency check failed (debug build)"
    assert swa.swa_status_string(99) == "unknown status"


NULL = None
P = ctypes.c_void_p
FAKE = ctypes.c_void_p(1 << 20)       # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def prefill(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, T=16, Hq=4, Hkv=2, d=64, W=4,
            scale=0.125, dt=1):
    return lib.swa_prefill(q, k, v, o, lse, B, T, Hq, Hkv, d, W, scale, dt, NULL)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=NULL), 1), (dict(o=NULL), 1), (dict(k=MISALIGNED), 1), (dict(Hq=3, Hkv=2), 1),
    (dict(W=0), 1), (dict(W=-5), 1), (dict(scale=0.0), 1), (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1), (dict(d=48), 2), (dict(d=256), 2), (dict(dt=7), 1),
    (dict(dt=0, d=130), 2), (dict(dt=0, d=6), 2), (dict(B=-1), 1), (dict(Hkv=0), 1),
])
def test_prefill_rejects(lib, kw, expect):
    assert prefill(lib, **kw) == expect


def test_prefill_empty_is_ok_without_touching_memory(lib):
    # B == 0 or T == 0: nothing to do, even with null pointers
    assert prefill(lib, q=NULL, k=NULL, v=NULL, o=NULL, B=0) == 0
    assert prefill(lib, q=NULL, k=NULL, v=NULL, o=NULL, T=0) == 0


def test_prefill_global_rejects(lib):
    f = lib.swa_prefill_global
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, NULL, 3, 1, 16, 2, 2, 64, 8, 0.125, 1, NULL) == 1  # g>0, no idx
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, FAKE, 17, 1, 16, 2, 2, 64, 8, 0.125, 1, NULL) == 1  # g > T
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, FAKE, -1, 1, 16, 2, 2, 64, 8, 0.125, 1, NULL) == 1
    assert f(NULL, NULL, NULL, NULL, NULL, NULL, 0, 0, 16, 2, 2, 64, 8, 0.125, 1, NULL) == 0


def test_prefill_chunk_rejects(lib):
    f = lib.swa_prefill_chunk
    call = lambda kc=FAKE, vc=FAKE, pos=FAKE, B=1, n=16, Hq=4, Hkv=2, d=64, W=32, dt=1: f(
        FAKE, FAKE, FAKE, FAKE, NULL, kc, vc, pos, B, n, Hq, Hkv, d, W, 0.125, dt, NULL)
    assert call(pos=NULL) == 1
    assert call(kc=NULL) == 1
    assert call(vc=MISALIGNED) == 1
    assert call(pos=ctypes.c_void_p((1 << 20) + 2)) == 1   # int32 positions need 4-byte alignment
    assert call(W=0) == 1
    assert call(d=48) == 2
    assert call(Hq=3) == 1
    assert call(n=0, kc=NULL, vc=NULL, pos=NULL) == 0
    assert call(B=0, kc=NULL, vc=NULL, pos=NULL) == 0


def test_sinks_reject(lib):
    f = lib.swa_prefill_sinks
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, -1, 1, 16, 4, 2, 64, 8, 0.125, 1, NULL) == 1   # negative sinks
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, 2, 1, 16, 4, 2, 48, 8, 0.125, 1, NULL) == 2    # d
    assert f(NULL, NULL, NULL, NULL, NULL, 2, 0, 16, 4, 2, 64, 8, 0.125, 1, NULL) == 0     # B == 0
    g = lib.swa_decode_sinks
    need = lib.swa_decode_workspace_bytes(64, 32, 8, 128, 4096)
    call = lambda ks=FAKE, vs=FAKE, n=4: g(FAKE, FAKE, FAKE, ks, vs, n, FAKE, NULL, FAKE, 64, 32, 8, 128, 4096,
                                          0.088, 1, FAKE, need, NULL)
    assert call(n=-1) == 1
    assert call(ks=NULL) == 1
    assert call(vs=MISALIGNED) == 1


def test_dilated_rejects(lib):
    f = lib.swa_prefill_dilated
    need = lib.swa_prefill_dilated_workspace_bytes(2, 300, 8, 2, 64, 3, 1, 0)
    assert need > 0
    assert lib.swa_prefill_dilated_workspace_bytes(2, 300, 8, 2, 64, 1, 1, 0) == 0   # dil 1: none
    call = lambda dil=3, sym=0, ws=FAKE, wsb=need: f(FAKE, FAKE, FAKE, FAKE, NULL, dil, sym, 2, 300, 8, 2, 64, 16,
                                                     0.125, 1, ws, wsb, NULL)
    assert call(dil=0) == 1
    assert call(sym=2) == 1
    assert call(ws=NULL) == 1
    assert call(wsb=need - 1) == 1
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == 1      # workspace needs 256-byte alignment


def test_varlen_rejects(lib):
    f = lib.swa_prefill_varlen
    call = lambda cu=FAKE, nseq=3, total=300, maxl=128, d=64, win=NULL: f(FAKE, FAKE, FAKE, FAKE, NULL, cu, win, nseq,
                                                                          total, maxl, 8, 2, d, 64, 0.125, 1, NULL)
    assert call(cu=NULL) == 1
    assert call(cu=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert call(nseq=-1) == 1
    assert call(maxl=301) == 1
    assert call(d=48) == 2
    assert call(win=ctypes.c_void_p((1 << 20) + 2)) == 1     # int32 windows need 4-byte alignment
    assert call(nseq=0, cu=NULL) == 0
    assert f(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 2, 0, 0, 8, 2, 64, 64, 0.125, 1, NULL) == 0   # no rows


def test_append_rejects(lib):
    f = lib.swa_cache_append
    assert f(FAKE, FAKE, FAKE, FAKE, NULL, NULL, 2, 1, 8, 128, 64, 1, NULL) == 1      # no pos
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 2, 1, 8, 4, 64, 1, NULL) == 2        # 8-byte rows
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 2, 1, 8, 128, 0, 1, NULL) == 1       # W = 0
    assert f(FAKE, MISALIGNED, FAKE, FAKE, FAKE, NULL, 2, 1, 8, 128, 64, 1, NULL) == 1
    assert f(NULL, NULL, NULL, NULL, NULL, NULL, 2, 0, 8, 128, 64, 1, NULL) == 0      # n == 0


def test_decode_rejects(lib):
    f = lib.swa_decode
    need = lib.swa_decode_workspace_bytes(2, 32, 8, 128, 4096)     # 32 splits: beyond one cluster
    assert need > 0
    args = lambda **kw: dict(dict(q=FAKE, kc=FAKE, vc=FAKE, o=FAKE, lse=NULL, pos=FAKE, B=2, Hq=32,
                                  Hkv=8, d=128, W=4096, scale=0.088, dt=1, ws=FAKE, wsb=need), **kw)
    call = lambda a: f(a["q"], a["kc"], a["vc"], a["o"], a["lse"], a["pos"], a["B"], a["Hq"], a["Hkv"],
                       a["d"], a["W"], a["scale"], a["dt"], a["ws"], a["wsb"], NULL)
    assert call(args(ws=NULL)) == 1
    assert call(args(wsb=need - 1)) == 1
    assert call(args(Hq=24, Hkv=8)) == 2      # group of 3
    assert call(args(Hq=36, Hkv=8)) == 1      # not divisible
    assert call(args(d=96)) == 2
    assert call(args(pos=NULL)) == 1
    assert call(args(B=0, q=NULL, kc=NULL, vc=NULL, o=NULL, pos=NULL)) == 0


def test_mask_export_rejects(lib):
    f = lib.swa_mask_export
    assert f(FAKE, 70000, 4, 0, NULL, 0, NULL) == 1
    assert f(FAKE, 16, 4, 0, FAKE, 2, NULL) == 1      # globals need the symmetric mode
    assert f(FAKE, 16, 4, 2, NULL, 0, NULL) == 1
    assert f(NULL, 0, 4, 0, NULL, 0, NULL) == 0


def test_debug_hook_rejects_bad_limits(lib):
    assert lib.swa_debug_expire_wait(0, NULL) == 1
    assert lib.swa_debug_expire_wait(10**8, NULL) == 1


def test_workspace_sizes(lib):
    # no workspace when one split suffices; otherwise [B,Hq,S,d+2] fp32
    assert lib.swa_decode_workspace_bytes(64, 32, 8, 128, 4096) == 64 * 32 * 8 * 130 * 4   # 8 splits
    assert lib.swa_decode_workspace_bytes(2, 32, 8, 128, 4096) == 2 * 32 * 32 * 130 * 4   # 32 splits
    assert lib.swa_decode_workspace_bytes(5, 32, 8, 128, 200) == 0        # one split (W < 256)
    assert lib.swa_decode_workspace_bytes(0, 32, 8, 128, 4096) == 0


def test_paged_rejects(lib):
    f = lib.swa_cache_append_paged
    call = lambda tbl=FAKE, P=16, W=64, npg=8, d=64, pos=FAKE: f(FAKE, FAKE, FAKE, FAKE, pos, tbl, NULL, 2, 1, 2, d,
                                                                 W, P, npg, 1, NULL)
    assert call(tbl=NULL) == 1
    assert call(P=12) == 1          # not a power of two
    assert call(P=128) == 1         # does not divide W
    assert call(P=0) == 1
    assert call(npg=0) == 1
    assert call(d=4) == 2           # 8-byte rows
    assert call(tbl=ctypes.c_void_p((1 << 20) + 2)) == 1
    g = lib.swa_decode_paged
    need = lib.swa_decode_workspace_bytes(64, 32, 8, 128, 4096)
    dcall = lambda tbl=FAKE, P=16, npg=16384, B=64: g(FAKE, FAKE, FAKE, tbl, FAKE, NULL, FAKE, B, 32, 8, 128, 4096,
                                                      P, npg, 0.088, 1, FAKE, need, NULL)
    assert dcall(tbl=NULL) == 1
    assert dcall(P=24) == 1
    assert dcall(npg=0) == 1
    assert dcall(B=0, tbl=NULL) == 0


def test_debug_build_exports_the_same_calls():
    import subprocess
    path = swa_build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in names, name

def test_backward_rejects(lib):
    f = lib.swa_prefill_backward
    need = lib.swa_prefill_backward_workspace_bytes(2, 300, 8)
    assert need == (2 * 300 * 8 * 4 + 255) // 256 * 256
    call = lambda sym=0, d=128, dt=1, ws=FAKE, wsb=need, lse=FAKE, W=64: f(FAKE, FAKE, FAKE, FAKE, lse, FAKE, FAKE,
                                                                             FAKE, FAKE, sym, 2, 300, 8, 2, d, W,
                                                                             0.088, dt, ws, wsb, NULL)
    assert call(dt=0) == 2           # fp32: no backward kernel
    assert call(d=32) == 2
    assert call(sym=2) == 1
    assert call(W=0) == 1
    assert call(wsb=need - 1) == 1
    assert call(ws=NULL) == 1
    assert call(lse=NULL) == 1
    assert call(lse=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert f(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 0, 300, 8, 2, 128, 64, 0.088, 1, NULL, 0,
             NULL) == 0      # B == 0
