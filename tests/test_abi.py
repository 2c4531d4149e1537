"""The C ABI on the CPU: the library builds for sm_100a, loads, exports every
entry point include/fp4q.h declares, and rejects bad arguments on the host
with the documented status codes before touching a device."""
import ctypes
import os
import re

import pytest

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp4q.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return fq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["fp4q_amax", "fp4q_quantize_nvfp4", "fp4q_quantize_mxfp4", "fp4q_quantize_2d",
              "fp4q_rht_amax", "fp4q_quantize_rht_sr", "fp4q_quantize_if4", "fp4q_dequantize",
              "fp4q_scale_bytes", "fp4q_workspace_bytes", "fp4q_status_string", "fp4q_version",
              "fp4q_quantize_mxfp6", "fp4q_gemm_nvfp4", "fp4q_quantize_if6",
              "fp4q_gemm_if4_nvfp4", "fp4q_quantize_if3"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_constants(L):
    assert fq.fp4q_status_string(0) == "FP4Q_OK"
    assert fq.fp4q_status_string(2) == "FP4Q_ERR_UNSUPPORTED_SHAPE"
    assert fq.fp4q_status_string(99) == "FP4Q_ERR_UNKNOWN"
    assert "sm_100a" in fq.fp4q_version()
    assert fq.fp4q_workspace_bytes() >= 4
    assert fq.fp4q_workspace_bytes(8192, 4096) == fq.fp4q_workspace_bytes(16, 16) >= 4
    assert fq.fp4q_workspace_bytes(-1, 16) == 0


def test_scale_bytes(L):
    assert fq.fp4q_scale_bytes(8192, 4096, 16, fq.SCALE_LINEAR) == 8192 * 256
    assert fq.fp4q_scale_bytes(8192, 4096, 16, fq.SCALE_SWIZZLED) == 8192 * 256
    assert fq.fp4q_scale_bytes(130, 80, 16, fq.SCALE_SWIZZLED) == 256 * 8
    assert fq.fp4q_scale_bytes(130, 80, 16, fq.SCALE_LINEAR) == 130 * 5
    assert fq.fp4q_scale_bytes(16, 24, 16, fq.SCALE_LINEAR) == 0      # cols % block
    assert fq.fp4q_scale_bytes(16, 32, 16, 7) == 0                    # bad layout


FAKE = ctypes.c_void_p(0x7F0000000000)          # 16-byte aligned, never dereferenced


def nv(L, **kw):
    a = dict(x=FAKE, dtype=0, rows=32, cols=64, ld=64, layouts=1, round=0, seed=0, amax=FAKE,
             s=FAKE, q_row=FAKE, sf_row=FAKE, q_col=FAKE, sf_col=FAKE, layout=0, ws=None,
             ws_bytes=0, stream=None)
    a.update(kw)
    return L.fp4q_quantize_nvfp4(a["x"], a["dtype"], a["rows"], a["cols"], a["ld"], a["layouts"],
                                 a["round"], a["seed"], a["amax"], a["s"], a["q_row"],
                                 a["sf_row"], a["q_col"], a["sf_col"], a["layout"], a["ws"],
                                 a["ws_bytes"], a["stream"])


def test_host_side_argument_checks(L):
    assert nv(L, dtype=5) == 1                       # bad dtype
    assert nv(L, ld=32) == 1                         # ld < cols
    assert nv(L, layouts=0) == 1 and nv(L, layouts=4) == 1
    assert nv(L, round=2) == 1
    assert nv(L, layout=3) == 1
    assert nv(L, cols=24, ld=24) == 2                # cols % 16
    assert nv(L, rows=24, layouts=2) == 2            # COLWISE needs rows % 16
    assert nv(L, layout=1) == 2                      # swizzle needs rows % 128
    assert nv(L, x=ctypes.c_void_p(0x7F0000000008)) == 3
    assert nv(L, ld=68) == 3                         # row stride not 16-byte aligned (BF16)
    assert nv(L, q_row=None) == 1
    assert L.fp4q_quantize_mxfp4(FAKE, 0, 32, 48, 48, 1, 0, FAKE, FAKE, None, None, 0, None) == 2
    assert L.fp4q_quantize_mxfp4(FAKE, 0, 32, 64, 64, 1, 9, FAKE, FAKE, None, None, 0, None) == 1
    assert L.fp4q_quantize_2d(FAKE, 1, 24, 64, 64, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0,
                              None, 0, None) == 2
    assert L.fp4q_quantize_rht_sr(FAKE, 0, 128, 64, 64, 32, 1, 0, FAKE, FAKE, FAKE, FAKE, 0,
                                  None, None, 0, None) == 1      # n must be 16 or 128
    assert L.fp4q_quantize_rht_sr(FAKE, 0, 120, 64, 64, 16, 1, 0, FAKE, FAKE, FAKE, FAKE, 0,
                                  None, None, 0, None) == 2      # tokens % n
    assert L.fp4q_quantize_rht_sr(FAKE, 0, 128, 68, 72, 16, 1, 0, FAKE, FAKE, FAKE, FAKE, 0,
                                  None, None, 0, None) == 2      # cols % 8
    assert L.fp4q_quantize_if4(FAKE, 0, 16, 40, 40, FAKE, FAKE, FAKE, FAKE, 0, None, 0, None) == 2
    assert L.fp4q_quantize_if4(FAKE, 0, 16, 48, 52, FAKE, FAKE, FAKE, FAKE, 0, None, 0, None) == 3
    assert L.fp4q_dequantize(0, FAKE, FAKE, 0, 1, 32, FAKE, 16, 64, FAKE, 1, None) == 1
    assert L.fp4q_dequantize(1, FAKE, FAKE, 0, 1, 32, None, 16, 48, FAKE, 1, None) == 2
    assert L.fp4q_dequantize(0, FAKE, FAKE, 0, 1, 16, None, 16, 64, FAKE, 1, None) == 1


def test_host_side_argument_checks_of_the_added_calls(L):
    # four-over-six: the NVFP4 rules
    f46 = lambda **kw: L.fp4q_quantize_four_over_six(
        kw.get("x", FAKE), 0, kw.get("rows", 32), kw.get("cols", 64), kw.get("ld", 64),
        kw.get("layouts", 1), FAKE, FAKE, kw.get("q_row", FAKE), FAKE, FAKE, FAKE,
        kw.get("layout", 0), None, 0, None)
    assert f46(layouts=0) == 1
    assert f46(cols=24, ld=24) == 2
    assert f46(rows=24, layouts=2) == 2
    assert f46(layout=1) == 2
    assert f46(q_row=ctypes.c_void_p(0x7F0000000008)) == 3
    assert f46(q_row=None) == 1
    # NVINT4: the IF4 rules
    assert L.fp4q_quantize_nvint4(FAKE, 0, 16, 40, 40, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                                  None) == 2
    assert L.fp4q_quantize_nvint4(FAKE, 0, 16, 48, 52, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                                  None) == 3
    assert L.fp4q_quantize_nvint4(FAKE, 0, 16, 48, 48, FAKE, FAKE, FAKE, FAKE, 5, None, 0,
                                  None) == 1
    # backward: RHT rules plus cols % 16 and both outputs
    bw = lambda **kw: L.fp4q_quantize_backward(
        FAKE, 0, kw.get("tokens", 128), kw.get("cols", 64), kw.get("ld", 64), kw.get("n", 16),
        kw.get("round", 1), 0, 1, FAKE, FAKE, FAKE, FAKE, kw.get("q_row", FAKE), FAKE,
        kw.get("q_t", FAKE), FAKE, kw.get("layout", 0), None, 0, None)
    assert bw(n=32) == 1
    assert bw(round=3) == 1
    assert bw(tokens=120) == 2
    assert bw(cols=72, ld=72) == 2                  # the row-wise output needs cols % 16
    assert bw(q_row=None) == 1 and bw(q_t=None) == 1
    assert bw(q_t=ctypes.c_void_p(0x7F0000000004)) == 3
    assert bw(layout=1, tokens=128, cols=64) == 2   # swizzled dY^T scales need cols % 128
    assert L.fp4q_quantize_nvfp4_noalloc(FAKE, 0, 32, 24, 24, 1, 0, 0, FAKE, FAKE, FAKE, FAKE,
                                         None, None, 0, None) == 2
    # MXFP6: cols % 32, the FP6 format and E8M0 mode, 16-byte aligned codes
    m6 = lambda **kw: L.fp4q_quantize_mxfp6(
        kw.get("x", FAKE), kw.get("dtype", 0), kw.get("rows", 32), kw.get("cols", 64),
        kw.get("ld", 64), kw.get("fmt", 0), kw.get("mode", 0), kw.get("q", FAKE), FAKE,
        kw.get("layout", 0), None)
    assert m6(fmt=2) == 1 and m6(fmt=-1) == 1
    assert m6(mode=3) == 1
    assert m6(layout=2) == 1
    assert m6(cols=48, ld=48) == 2
    assert m6(layout=1) == 2                        # swizzle needs rows % 128
    assert m6(rows=128, cols=96, ld=96, layout=1) == 2   # and (cols/32) % 4
    assert m6(ld=60) == 1                           # ld < cols
    assert m6(x=ctypes.c_void_p(0x7F0000000008)) == 3
    assert m6(q=ctypes.c_void_p(0x7F0000000008)) == 3
    assert m6(q=None) == 1
    assert m6(rows=0) == 0                          # nothing to do, nothing touched
    # GEMM: 128x128 output tiles, K % 256, aligned operands
    gm = lambda **kw: L.fp4q_gemm_nvfp4(
        kw.get("qa", FAKE), FAKE, None, FAKE, FAKE, None, kw.get("M", 128), kw.get("N", 128),
        kw.get("K", 256), kw.get("c", FAKE), kw.get("dt", 1), kw.get("ldc", 128), None, None)
    assert gm(dt=3) == 1
    assert gm(ldc=64) == 1
    assert gm(M=96) == 2 and gm(N=200, ldc=200) == 2 and gm(K=128) == 2
    assert gm(c=ctypes.c_void_p(0x7F0000000008)) == 3
    assert gm(ldc=130) == 3                         # row stride not 16-byte aligned (FP32)
    assert gm(qa=None) == 1
    assert gm(qa=ctypes.c_void_p(0x7F0000000004)) == 3
    assert gm(M=0) == 0
    # the IF4 GEMM: GEMM shapes plus a workspace of the stated size
    assert L.fp4q_gemm_if4_workspace_bytes(128, 256) == 3 * 128 * 128 + 128 * 16
    g4 = lambda **kw: L.fp4q_gemm_if4_nvfp4(
        FAKE, FAKE, None, FAKE, FAKE, None, kw.get("M", 128), 128, kw.get("K", 256), FAKE, 128,
        kw.get("ws", FAKE), kw.get("wsb", 1 << 20), None, None)
    assert g4(K=128) == 2 and g4(M=96) == 2
    assert g4(wsb=100) == 4 and g4(ws=None) == 4
    assert g4(ws=ctypes.c_void_p(0x7F0000000008)) == 3
    # the test hook wants a status pointer and some K
    assert L.fp4q_gemm_nvfp4_withhold_loads(FAKE, FAKE, None, FAKE, FAKE, None, 128, 128, 256,
                                            FAKE, 1, 128, None, None) == 1
    # IF6: the IF4 rules
    assert L.fp4q_quantize_if6(FAKE, 0, 16, 40, 40, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                               None) == 2
    assert L.fp4q_quantize_if6(FAKE, 0, 16, 48, 52, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                               None) == 3
    assert L.fp4q_quantize_if6(FAKE, 0, 16, 48, 48, FAKE, FAKE, FAKE, FAKE, 4, None, 0,
                               None) == 1
    assert L.fp4q_quantize_if6(FAKE, 0, 16, 48, 48, FAKE, FAKE, None, FAKE, 0, None, 0,
                               None) == 1
    assert L.fp4q_dequantize(5, FAKE, FAKE, 0, 1, 32, FAKE, 16, 64, FAKE, 1, None) == 1
    assert L.fp4q_dequantize(5, FAKE, FAKE, 0, 1, 16, None, 16, 64, FAKE, 1, None) == 1
    # dequantize: MXFP6 formats take 1x32 blocks and no tensor scale
    assert L.fp4q_dequantize(3, FAKE, FAKE, 0, 1, 16, None, 16, 64, FAKE, 1, None) == 1
    assert L.fp4q_dequantize(4, FAKE, FAKE, 0, 1, 32, None, 16, 48, FAKE, 1, None) == 2
    assert L.fp4q_dequantize(7, FAKE, FAKE, 0, 1, 16, FAKE, 16, 64, FAKE, 1, None) == 1
    # IF3: the IF4 rules, 1x16 blocks with a tensor scale
    assert L.fp4q_quantize_if3(FAKE, 0, 16, 40, 40, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                               None) == 2
    assert L.fp4q_quantize_if3(FAKE, 0, 16, 48, 52, FAKE, FAKE, FAKE, FAKE, 0, None, 0,
                               None) == 3
    assert L.fp4q_quantize_if3(FAKE, 0, 16, 48, 48, FAKE, FAKE, FAKE, FAKE, 4, None, 0,
                               None) == 1
    assert L.fp4q_quantize_if3(FAKE, 0, 16, 48, 48, FAKE, FAKE, None, FAKE, 0, None, 0,
                               None) == 1
    assert L.fp4q_quantize_if3(FAKE, 0, 16, 48, 48, FAKE, FAKE,
                               ctypes.c_void_p(0x7F0000000008), FAKE, 0, None, 0, None) == 3
    assert L.fp4q_dequantize(6, FAKE, FAKE, 0, 1, 32, FAKE, 16, 64, FAKE, 1, None) == 1
    assert L.fp4q_dequantize(6, FAKE, FAKE, 0, 1, 16, None, 16, 64, FAKE, 1, None) == 1
    assert L.fp4q_dequantize(6, FAKE, FAKE, 0, 1, 16, FAKE, 16, 40, FAKE, 1, None) == 2


def test_python_binding_refuses_cpu_tensors(L):
    import torch
    with pytest.raises(ValueError):
        fq.fp4q_quantize_nvfp4(torch.zeros(16, 16, dtype=torch.bfloat16))


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp4q.h"
int main(void) {
  if (strstr(fp4q_version(), "sm_100a") == NULL) return 2;
  if (fp4q_scale_bytes(130, 80, 16, FP4Q_SCALE_SWIZZLED_128x4) != 256 * 8) return 3;
  if (strcmp(fp4q_status_string(FP4Q_ERR_MISALIGNED), "FP4Q_ERR_MISALIGNED") != 0) return 4;
  /* an argument error is returned before anything touches a device */
  if (fp4q_quantize_if3(NULL, FP4Q_BF16, 16, 48, 48, NULL, NULL, NULL, NULL,
                        FP4Q_SCALE_LINEAR, NULL, 0, NULL) != FP4Q_ERR_INVALID_ARG) return 5;
  puts("ok");
  return 0;
}
"""


@pytest.mark.parametrize("compiler", [["gcc", "-std=c99", "-x", "c"],
                                      ["g++", "-std=c++17", "-x", "c++"]])
def test_header_is_plain_c_and_links(L, tmp_path, compiler):
    """The public header compiles as strict C99 and as C++ (extern "C"), and a
    program linked against the library runs its host-side calls."""
    import subprocess
    src = tmp_path / "use_fp4q.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_fp4q"
    libdir = os.path.dirname(fq.library_path)
    subprocess.check_call([*compiler, "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), str(src), "-x", "none",
                           "-L", libdir, "-lfp4q", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)


def test_binding_declares_every_header_function():
    """The Python binding gives every entry point of the header a ctypes
    signature, and none that the header lacks."""
    src = open(os.path.join(ROOT, "fp4_block_scaled_04_b200", "__init__.py")).read()
    bound = set(re.findall(r'"(fp4q_\w+)":\s*\(', src))
    assert bound == set(declared_functions())


def test_noalloc_rejects_what_the_workspace_call_rejects(L):
    """The no-allocation call checks its arguments exactly as
    fp4q_quantize_nvfp4 does, before it looks at any device: with amax NULL
    (the path that would otherwise look up its scratch array first) every
    rejected call returns the workspace call's status.  No GPU is needed,
    because nothing past the checks runs."""
    def both(**kw):
        a = (kw.get("x", FAKE), kw.get("dtype", 0), kw.get("rows", 32), kw.get("cols", 64),
             kw.get("ld", 64), kw.get("layouts", 3), kw.get("round", 0), 0, None, FAKE,
             kw.get("q_row", FAKE), FAKE, kw.get("q_col", FAKE), FAKE, kw.get("layout", 0))
        return (L.fp4q_quantize_nvfp4_noalloc(*a, None),
                L.fp4q_quantize_nvfp4(*a, FAKE, 256, None))
    cases = [dict(dtype=7), dict(layouts=0), dict(layouts=4), dict(round=2), dict(layout=5),
             dict(cols=24, ld=24), dict(rows=24), dict(ld=60), dict(layout=1),
             dict(q_row=ctypes.c_void_p(0x7F0000000008)), dict(q_col=None),
             dict(x=ctypes.c_void_p(0x7F0000000004))]
    for kw in cases:
        got, want = both(**kw)
        assert want != 0, kw
        assert got == want, (kw, got, want)
