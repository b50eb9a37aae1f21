"""C-ABI checks that need no GPU: the library builds and loads, exports every symbol declared in
include/*.h, and rejects bad arguments with the documented status codes before touching a device.

Fake pointers are used only in cases that fail validation before the device check, so no test here
can ever reach a kernel launch, with or without a GPU.
"""
import ctypes
import glob
import os
import re

import pytest

from conftest import ROOT

import exact_tiled_attention_47_b200 as fa
from exact_tiled_attention_47_b200 import build as fabuild


@pytest.fixture(scope="module")
def lib():
    fabuild.build()
    return fa._lib.load()


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(fa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("fa_fwd", "fa_decode_splitkv", "fa_decode_workspace_bytes", "fa_status_string",
              "fa_device_status", "fa_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n
        assert n in fa._lib.SIGNATURES, f"binding has no signature for {n}"


def test_binding_names_match_c_names():
    for n in _declared_functions():
        assert callable(getattr(fa, n)), n


def test_abi_version_and_status_strings(lib):
    assert fa.fa_abi_version() == 1
    seen = set()
    for code in range(13):
        s = fa.fa_status_string(code)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 13
    assert fa.fa_status_string(999) == "unknown status"
    assert fa.fa_build_flags() == 0  # the release library


def test_debug_library_builds_and_exports_the_same_boundary():
    from exact_tiled_attention_47_b200 import build
    path = build.build(debug=True)
    dbg = fa._lib.load(path)
    assert dbg.fa_build_flags() == fa.FA_BUILD_DEBUG
    for n in _declared_functions():
        assert hasattr(dbg, n), n


def test_workspace_bytes(lib):
    B, H, D, S = 64, 32, 128, 16
    exp = S * B * H * (D + 1) * 4
    got = fa.fa_decode_workspace_bytes(B, H, D, S)
    assert got >= exp and got % 256 == 0 and got - exp < 256
    assert fa.fa_decode_workspace_bytes(0, H, D, S) == 0
    assert fa.fa_decode_workspace_bytes(B, H, 96, S) == 0
    assert fa.fa_decode_workspace_bytes(B, H, D, 0) == 0


A = 0x100000  # a 16-byte aligned fake address (never dereferenced: every case fails validation)


def _fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, Nq=128, Nk=128, D=64, scale=0.125, causal=0,
         cu=None, in_dtype=0, o_dtype=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, D, scale, causal, cu, None, in_dtype, o_dtype)


def test_fwd_validation_codes(lib):
    assert _fwd(lib, q=None) == fa.FA_ERR_NULL
    assert _fwd(lib, lse=None) == fa.FA_ERR_NULL
    assert _fwd(lib, in_dtype=2) == fa.FA_ERR_DTYPE          # fp32 inputs rejected
    assert _fwd(lib, in_dtype=5) == fa.FA_ERR_DTYPE
    assert _fwd(lib, in_dtype=0, o_dtype=1) == fa.FA_ERR_DTYPE  # bf16 in, fp16 out
    assert _fwd(lib, D=32) == fa.FA_ERR_HEADDIM
    assert _fwd(lib, D=96) == fa.FA_ERR_HEADDIM
    assert _fwd(lib, D=256) == fa.FA_ERR_HEADDIM
    assert _fwd(lib, B=0) == fa.FA_ERR_SHAPE
    assert _fwd(lib, Nk=0) == fa.FA_ERR_SHAPE
    assert _fwd(lib, Nq=0) == fa.FA_ERR_SHAPE
    assert _fwd(lib, scale=0.0) == fa.FA_ERR_SHAPE
    assert _fwd(lib, scale=-1.0) == fa.FA_ERR_SHAPE
    assert _fwd(lib, scale=float("nan")) == fa.FA_ERR_SHAPE
    assert _fwd(lib, scale=float("inf")) == fa.FA_ERR_SHAPE
    assert _fwd(lib, B=70000) == fa.FA_ERR_SHAPE
    assert _fwd(lib, B=200, Nq=1 << 24) == fa.FA_ERR_SHAPE
    assert _fwd(lib, cu=A, Nq=100, Nk=200) == fa.FA_ERR_SHAPE  # varlen needs one packed extent
    assert _fwd(lib, q=A + 8) == fa.FA_ERR_ALIGN
    assert _fwd(lib, o=A + 2) == fa.FA_ERR_ALIGN
    assert _fwd(lib, lse=A + 2) == fa.FA_ERR_ALIGN
    assert _fwd(lib, cu=A + 2) == fa.FA_ERR_ALIGN


def test_fwd_prefix_validation_codes(lib):
    def pre(prefix, **kw):
        a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, Nq=128, Nk=128, D=64, scale=0.125, cu=None)
        a.update(kw)
        return lib.fa_fwd_prefix(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"], a["Nk"],
                                 a["D"], a["scale"], prefix, a["cu"], None, 0, 0)
    assert pre(-1) == fa.FA_ERR_SHAPE
    assert pre(10, q=None) == fa.FA_ERR_NULL
    assert pre(10, D=96) == fa.FA_ERR_HEADDIM
    assert pre(10, scale=0.0) == fa.FA_ERR_SHAPE
    assert pre(10, o=A + 2) == fa.FA_ERR_ALIGN


def _dec(lib, q=A, k=A, v=A, o=A, lse=A, B=2, H=2, Nk=64, D=128, scale=0.1, S=4, ws=A,
         wsb=1 << 20, in_dtype=0, o_dtype=0):
    return lib.fa_decode_splitkv(q, k, v, o, lse, B, H, Nk, D, scale, S, ws, wsb, None, in_dtype, o_dtype)


def test_decode_validation_codes(lib):
    assert _dec(lib, k=None) == fa.FA_ERR_NULL
    assert _dec(lib, in_dtype=2) == fa.FA_ERR_DTYPE
    assert _dec(lib, o_dtype=1) == fa.FA_ERR_DTYPE
    assert _dec(lib, D=80) == fa.FA_ERR_HEADDIM
    assert _dec(lib, Nk=0) == fa.FA_ERR_SHAPE
    assert _dec(lib, S=0) == fa.FA_ERR_SHAPE
    assert _dec(lib, S=129) == fa.FA_ERR_SHAPE
    assert _dec(lib, scale=0.0) == fa.FA_ERR_SHAPE
    assert _dec(lib, v=A + 4) == fa.FA_ERR_ALIGN
    assert _dec(lib, ws=None) == fa.FA_ERR_WORKSPACE
    need = fa.fa_decode_workspace_bytes(2, 2, 128, 4)
    assert _dec(lib, wsb=need - 1) == fa.FA_ERR_WORKSPACE
    assert _dec(lib, ws=A + 8, wsb=need) == fa.FA_ERR_ALIGN


def test_decode_gqa_validation_codes(lib):
    def gqa(Hq=8, Hkv=2, sl=None, wsb=1 << 20, ws=A, **kw):
        a = dict(q=A, k=A, v=A, o=A, lse=A, B=2, Nk=64, D=128, scale=0.1, S=4)
        a.update(kw)
        return lib.fa_decode_splitkv_gqa(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], Hq, Hkv, a["Nk"], a["D"],
                                         a["scale"], a["S"], sl, ws, wsb, None, 0, 0)
    assert gqa(Hkv=0) == fa.FA_ERR_SHAPE
    assert gqa(Hkv=3) == fa.FA_ERR_SHAPE          # 8 query heads are not a multiple of 3
    assert gqa(Hq=2, Hkv=4) == fa.FA_ERR_SHAPE     # more KV heads than query heads
    assert gqa(sl=A + 2) == fa.FA_ERR_ALIGN
    assert gqa(q=None) == fa.FA_ERR_NULL
    need = fa.fa_decode_workspace_bytes(2, 8, 128, 4)  # sized by the query heads
    assert gqa(wsb=need - 1) == fa.FA_ERR_WORKSPACE


def _paged(lib, table=A, npg=32, ps=64, pps=4, B=2, Hq=8, Hkv=2, sl=None, ws=A, wsb=1 << 20, q=A, kp=A, D=128):
    return lib.fa_decode_splitkv_paged(q, kp, A, table, A, A, B, Hq, Hkv, npg, ps, pps, D, 0.1, 4, sl, ws, wsb,
                                       None, 0, 0)


def test_decode_paged_validation_codes(lib):
    assert _paged(lib, table=None) == fa.FA_ERR_NULL
    assert _paged(lib, q=None) == fa.FA_ERR_NULL
    for ps in (8, 48, 96, 1 << 17):        # page size: a power of two from 16 to 65536
        assert _paged(lib, ps=ps) == fa.FA_ERR_SHAPE, ps
    assert _paged(lib, npg=0) == fa.FA_ERR_SHAPE
    assert _paged(lib, pps=0) == fa.FA_ERR_SHAPE
    assert _paged(lib, npg=1 << 25, ps=64) == fa.FA_ERR_SHAPE    # pool rows reach 2^31
    assert _paged(lib, pps=1 << 25, ps=64) == fa.FA_ERR_SHAPE    # capacity reaches 2^31
    assert _paged(lib, Hkv=3) == fa.FA_ERR_SHAPE
    assert _paged(lib, D=96) == fa.FA_ERR_HEADDIM
    assert _paged(lib, kp=A + 8) == fa.FA_ERR_ALIGN
    assert _paged(lib, table=A + 2) == fa.FA_ERR_ALIGN
    assert _paged(lib, sl=A + 2) == fa.FA_ERR_ALIGN
    need = fa.fa_decode_workspace_bytes(2, 8, 128, 4)
    assert _paged(lib, wsb=need - 1) == fa.FA_ERR_WORKSPACE


def _shard(lib, part=A, q=A, Nk=64, off=0, tot=128, sl=None, ws=A, wsb=1 << 20, in_dtype=0):
    return lib.fa_decode_splitkv_shard(q, A, A, part, 2, 8, 2, Nk, off, tot, 128, 0.1, 4, sl, ws, wsb, None, in_dtype)


def _merge(lib, parts=A, R=2, B=2, H=8, D=128, o=A, lse=A, o_dtype=0):
    return lib.fa_decode_merge(parts, R, B, H, D, o, lse, None, o_dtype)


def test_decode_shard_and_merge_validation_codes(lib):
    assert _shard(lib, part=None) == fa.FA_ERR_NULL
    assert _shard(lib, q=None) == fa.FA_ERR_NULL
    assert _shard(lib, off=-1) == fa.FA_ERR_SHAPE
    assert _shard(lib, off=65) == fa.FA_ERR_SHAPE        # keys 65..128 run past a 128-key cache
    assert _shard(lib, tot=0) == fa.FA_ERR_SHAPE
    assert _shard(lib, Nk=0) == fa.FA_ERR_SHAPE
    assert _shard(lib, in_dtype=2) == fa.FA_ERR_DTYPE
    assert _shard(lib, part=A + 4) == fa.FA_ERR_ALIGN
    assert _shard(lib, sl=A + 2) == fa.FA_ERR_ALIGN
    assert _shard(lib, wsb=fa.fa_decode_workspace_bytes(2, 8, 128, 4) - 1) == fa.FA_ERR_WORKSPACE
    assert _merge(lib, parts=None) == fa.FA_ERR_NULL
    assert _merge(lib, lse=None) == fa.FA_ERR_NULL
    assert _merge(lib, o_dtype=3) == fa.FA_ERR_DTYPE
    assert _merge(lib, D=96) == fa.FA_ERR_HEADDIM
    assert _merge(lib, R=0) == fa.FA_ERR_SHAPE
    assert _merge(lib, B=0) == fa.FA_ERR_SHAPE
    assert _merge(lib, parts=A + 8) == fa.FA_ERR_ALIGN
    assert _merge(lib, o=A + 2) == fa.FA_ERR_ALIGN


def test_decode_part_bytes(lib):
    from exact_tiled_attention_47_b200.sharded import part_floats
    assert fa.fa_decode_part_bytes(2, 8, 128) == 2 * 8 * 129 * 4
    assert fa.fa_decode_part_bytes(3, 1, 64) == 784             # 3 * 65 * 4 = 780, padded to 16 bytes
    for B, H, D in ((2, 8, 128), (3, 1, 64), (7, 5, 64), (64, 32, 128)):
        assert fa.fa_decode_part_bytes(B, H, D) == 4 * part_floats(B, H, D)
    assert fa.fa_decode_part_bytes(0, 8, 128) == 0
    assert fa.fa_decode_part_bytes(2, 8, 96) == 0


def test_bwd_validation_codes(lib):
    def bwd(**kw):
        a = dict(q=A, k=A, v=A, o=A, do=A, lse=A, dq=A, dk=A, dv=A, B=1, H=1, Nq=128, Nk=128, D=64, scale=0.125,
                 causal=0, ws=A, wsb=1 << 20, in_dtype=0, g_dtype=0)
        a.update(kw)
        return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"], a["B"], a["H"],
                          a["Nq"], a["Nk"], a["D"], a["scale"], a["causal"], a["ws"], a["wsb"], None, a["in_dtype"],
                          a["g_dtype"])
    assert bwd(do=None) == fa.FA_ERR_NULL
    assert bwd(dv=None) == fa.FA_ERR_NULL
    assert bwd(in_dtype=2) == fa.FA_ERR_DTYPE
    assert bwd(g_dtype=1) == fa.FA_ERR_DTYPE
    assert bwd(D=96) == fa.FA_ERR_HEADDIM
    assert bwd(Nk=0) == fa.FA_ERR_SHAPE
    assert bwd(scale=-1.0) == fa.FA_ERR_SHAPE
    assert bwd(dk=A + 8) == fa.FA_ERR_ALIGN
    assert bwd(ws=None) == fa.FA_ERR_WORKSPACE
    assert bwd(wsb=fa.fa_bwd_workspace_bytes(1, 1, 128) - 1) == fa.FA_ERR_WORKSPACE
    assert fa.fa_bwd_workspace_bytes(2, 3, 100) == 2560  # 2*3*100*4 = 2400 rounded up to 256


def test_bwd_masked_validation_codes(lib):
    def bwd(**kw):
        a = dict(q=A, k=A, v=A, o=A, do=A, lse=A, dq=A, dk=A, dv=A, B=2, H=3, Nq=300, Nk=300, D=64, scale=0.125,
                 causal=1, prefix=0, cu=None, ws=A, wsb=1 << 20, in_dtype=0, g_dtype=0)
        a.update(kw)
        return lib.fa_bwd_masked(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                                 a["B"], a["H"], a["Nq"], a["Nk"], a["D"], a["scale"], a["causal"], a["prefix"],
                                 a["cu"], a["ws"], a["wsb"], None, a["in_dtype"], a["g_dtype"])
    assert bwd(lse=None) == fa.FA_ERR_NULL
    assert bwd(g_dtype=1) == fa.FA_ERR_DTYPE
    assert bwd(D=80) == fa.FA_ERR_HEADDIM
    assert bwd(prefix=-1) == fa.FA_ERR_SHAPE
    assert bwd(cu=A, Nk=299) == fa.FA_ERR_SHAPE          # varlen is self-attention: Nq == Nk
    assert bwd(cu=A + 2) == fa.FA_ERR_ALIGN
    assert bwd(q=A + 4) == fa.FA_ERR_ALIGN
    # varlen needs one row term per packed row and head: H * total floats, whatever B is
    need = fa.fa_bwd_workspace_bytes(1, 3, 300)
    assert bwd(cu=A, wsb=need - 1) == fa.FA_ERR_WORKSPACE
    assert bwd(cu=A, ws=None) == fa.FA_ERR_WORKSPACE
    assert bwd(wsb=fa.fa_bwd_workspace_bytes(2, 3, 300) - 1) == fa.FA_ERR_WORKSPACE


def test_device_status_null(lib):
    assert lib.fa_device_status(None, 0) == fa.FA_ERR_NULL


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU answer")
def test_no_device_is_reported(lib):
    # All arguments valid: the only failing check is the device one, and nothing is launched.
    assert _fwd(lib) == fa.FA_ERR_DEVICE
    assert lib.fa_fwd_prefix(A, A, A, A, A, 1, 1, 128, 128, 64, 0.125, 10, None, None, 0, 0) == fa.FA_ERR_DEVICE
    assert _dec(lib) == fa.FA_ERR_DEVICE
    w = ctypes.c_int(0)
    assert lib.fa_selftest_wait_timeout(ctypes.byref(w), None) == fa.FA_ERR_DEVICE
    assert lib.fa_bwd(A, A, A, A, A, A, A, A, A, 1, 1, 128, 128, 64, 0.125, 0, A, 1 << 20, None, 0, 0) == fa.FA_ERR_DEVICE
    assert lib.fa_bwd_masked(A, A, A, A, A, A, A, A, A, 2, 1, 300, 300, 64, 0.125, 1, 7, A, A, 1 << 20, None, 0,
                             0) == fa.FA_ERR_DEVICE
    assert lib.fa_decode_splitkv_gqa(A, A, A, A, A, 2, 8, 2, 64, 128, 0.1, 4, A, A, 1 << 20, None, 0, 0) == fa.FA_ERR_DEVICE
    assert _paged(lib) == fa.FA_ERR_DEVICE
    assert _paged(lib, ps=16, sl=A) == fa.FA_ERR_DEVICE
    assert _shard(lib) == fa.FA_ERR_DEVICE
    assert _shard(lib, off=64, sl=A) == fa.FA_ERR_DEVICE
    assert _merge(lib) == fa.FA_ERR_DEVICE
    assert _merge(lib, o_dtype=2) == fa.FA_ERR_DEVICE
    out = ctypes.c_int(0)
    assert lib.fa_device_status(ctypes.byref(out), 0) == fa.FA_ERR_DEVICE


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(fa.LibraryMissing):
        fa._lib.load(str(tmp_path / "nope.so"))


def test_plain_c_program(lib, tmp_path):
    """The boundary is usable from C99 alone: tests/c_abi_check.c compiled with gcc against
    include/fa.h and linked to the built library (no CUDA headers, no C++, no torch)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(fa.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    src = os.path.join(ROOT, "tests", "c_abi_check.c")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", libdir, "-lfa_sm100", "-Wl,-rpath," + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    import torch
    args = [] if torch.cuda.is_available() else ["nodevice"]
    r = subprocess.run([exe] + args, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c_abi_check: ok" in r.stdout
