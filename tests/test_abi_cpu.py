"""CPU checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments before enqueuing anything (no CUDA call is made on these
paths, so they run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

import decode_moe_layer_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P = ctypes.c_void_p


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    lib = moe.load()
    decl = declared_functions()
    assert decl, "no declarations found"
    for name in decl:
        assert hasattr(lib, name), name
    assert decl == set(moe.EXPORTS)


def test_status_strings():
    assert [moe.moe_status_string(s) for s in range(0, -6, -1)] == [
        "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED_SHAPE", "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA",
        "MOE_ERR_TIMEOUT"]
    assert moe.moe_status_string(7) == "MOE_ERR_UNKNOWN"


def test_workspace_bytes():
    a = moe.moe_workspace_bytes(8, 2048, 768, 128, 8)
    b = moe.moe_workspace_bytes(16, 2048, 768, 128, 8)
    assert 0 < a < b
    assert moe.moe_workspace_bytes(0, 2048, 768, 128, 8) > 0
    # the fp32 per-assignment rows dominate at large M: M*k*H*4 bytes
    big = moe.moe_workspace_bytes(1024, 4096, 1536, 128, 8)
    assert big >= 1024 * 8 * 4096 * 4
    for bad in [(8, 2047, 768, 128, 8), (8, 2048, 770, 128, 8), (8, 2048, 768, 4, 8), (8, 2048, 768, 2048, 8),
                (8, 2048, 768, 128, 33), (4096, 2048, 768, 128, 8), (-1, 2048, 768, 128, 8)]:
        assert moe.moe_workspace_bytes(*bad) == 0, bad


def _fwd_ex(lib, x=0x100000, out=0x200000, ws=0x300000, ws_bytes=1 << 40, M=8, H=2048, I=768, E=128, k=8,
            bias=None, ids=None):
    w = P(0x400000)
    return lib.moe_mxfp4_forward_ex(P(x), w, bias, w, w, w, w, P(out), M, H, I, E, k, ids, None, None,
                                    P(ws), ws_bytes, None)


def test_forward_ex_validation():
    lib = moe.load()
    assert _fwd_ex(lib, M=0) == moe.MOE_OK                       # M = 0: nothing enqueued
    assert _fwd_ex(lib, ws_bytes=100) == moe.MOE_ERR_WORKSPACE
    assert _fwd_ex(lib, x=0x100008) == moe.MOE_ERR_INVALID_ARG    # misaligned x
    assert _fwd_ex(lib, out=0x100000) == moe.MOE_ERR_INVALID_ARG  # out aliases x
    assert _fwd_ex(lib, ws=0x300010) == moe.MOE_ERR_INVALID_ARG   # workspace not 256-aligned
    assert _fwd_ex(lib, bias=P(0x500002)) == moe.MOE_ERR_INVALID_ARG
    assert _fwd_ex(lib, H=1000) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _fwd_ex(lib, k=0) == moe.MOE_ERR_INVALID_ARG
    assert _fwd_ex(lib, M=-3) == moe.MOE_ERR_INVALID_ARG
    assert _fwd_ex(lib, E=4, k=8) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert _fwd_ex(lib, M=4096) == moe.MOE_ERR_UNSUPPORTED_SHAPE   # M*k above the permutation limit
    assert lib.moe_mxfp4_forward_ex(None, P(16), None, P(16), P(16), P(16), P(16), P(32), 8, 2048, 768, 128, 8,
                                    None, None, None, P(256), 1 << 40, None) == moe.MOE_ERR_INVALID_ARG


def test_step_validation():
    lib = moe.load()
    a = P(0x1000)
    assert lib.moe_route(None, a, None, a, a, 1, 2048, 128, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(a, a, None, a, a, 0, 2048, 128, 8, None) == moe.MOE_OK
    assert lib.moe_route(P(0x1001), a, None, a, a, 1, 2048, 128, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(a, a, None, a, a, 1, 2048, 128, 33, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_permute(a, a, a, None, 4, 128, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(a, a, a, a, 0, 128, 8, None) == moe.MOE_OK
    assert lib.moe_permute(a, a, a, a, 4, 2000, 8, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_gate_up_swiglu(a, a, a, a, a, None, 4, 2048, 768, 128, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_up_swiglu(a, a, a, a, a, a, 4, 2048, 100, 128, 8, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_down_combine(a, a, a, a, a, a, None, 4, 2048, 768, 128, 8, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_down_combine(a, a, a, a, a, a, a, 0, 2048, 768, 128, 8, None) == moe.MOE_OK
    assert lib.moe_mxfp4_forward(a, a, a, a, a, a, a, 4, 2048, 768, 128, 8, None) == moe.MOE_ERR_INVALID_ARG


def test_selftest_validation():
    # argument checks only (no launch): null and misaligned status pointers are refused
    lib = moe.load()
    assert lib.moe_selftest_wait_timeout(None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(P(0x1002), None) == moe.MOE_ERR_INVALID_ARG


def test_forward_launch_counts():
    # 5 launches at decode sizes (fused select), 6 with the separate top-k + permutation, and 5
    # more (the gather and the small- and large-tile tensor-core GEMMs of both projections) once the
    # tensor-core path is on: H and I multiples of 512, M >= 5 and experts averaging >= 2.5
    # assignments; one fewer when down and the combine are one launch (I <= 1024, at most 8 tiles)
    lib = moe.load()
    assert lib.moe_forward_launches(0, 2048, 768, 128, 8) == 0
    assert lib.moe_forward_launches(1, 2048, 768, 128, 8) == 4
    assert lib.moe_forward_launches(2, 1024, 512, 16, 4) == 4
    assert lib.moe_forward_launches(8, 2048, 768, 128, 8) == 5
    assert lib.moe_forward_launches(1, 7168, 2048, 256, 8) == 5
    assert lib.moe_forward_launches(32, 7168, 2048, 256, 8) == 5
    assert lib.moe_forward_launches(96, 2048, 768, 128, 8) == 6
    assert lib.moe_forward_launches(256, 7168, 2048, 256, 8) == 11
    assert lib.moe_forward_launches(1024, 4096, 1536, 128, 8) == 11
    assert lib.moe_forward_launches(8, 2048, 100, 128, 8) == moe.MOE_ERR_UNSUPPORTED_SHAPE


def test_header_is_plain_c_and_links(tmp_path):
    # include/moe.h compiles as strict C99, every declared function resolves against libmoe.so, and
    # the host-only entry points answer from a C program (no torch, no GPU)
    names = sorted(declared_functions())
    checks = ("    typedef void (*fn)(void);\n    fn volatile table[] = {%s};\n"
              "    for (unsigned i = 0; i < sizeof(table) / sizeof(table[0]); ++i)\n"
              "        if (!table[i]) return 2;" % ", ".join("(fn)%s" % n for n in names))
    src = tmp_path / "abi.c"
    src.write_text("""#include "moe.h"
#include <stdio.h>
#include <string.h>
int main(void)
{
%s
    if (strcmp(moe_status_string(MOE_ERR_TIMEOUT), "MOE_ERR_TIMEOUT") != 0) return 3;
    if (moe_workspace_bytes(8, 2048, 768, 128, 8) == 0) return 4;
    if (moe_forward_launches(8, 2048, 768, 128, 8) != 5) return 5;
    if (moe_forward_launches(8, 2047, 768, 128, 8) != MOE_ERR_UNSUPPORTED_SHAPE) return 6;
    printf("ok\\n");
    return 0;
}
""" % checks)
    exe = str(tmp_path / "abi")
    libdir = os.path.dirname(moe.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", exe,
                           "-L", libdir, "-lmoe", "-Wl,-rpath," + libdir])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
