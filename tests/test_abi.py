"""The C-ABI library loads, exports every symbol the header declares, and
rejects invalid arguments on the host before touching a device (no GPU
needed)."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_accumulate_b200 import binding as B
from post_weight_quantization_accumulate_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_all_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    # and the binding covers exactly the header
    assert sorted(s[0] for s in B.SIGNATURES) == names


def test_version_status_strings(lib):
    assert B.gptq_version() >= 100
    assert B.gptq_status_string(0) == "ok"
    for s in range(1, 8):
        assert B.gptq_status_string(s) not in ("", "unknown status")
    assert B.gptq_status_string(99) == "unknown status"
    assert isinstance(B.gptq_launch_count(), int)


def test_workspace_bytes(lib):
    w = B.gptq_workspace_bytes(4096, 4096, 128)
    assert w >= 2 * 4096 * 4096 * 4          # factorisation: working copy and inverse
    assert w >= 4096 * 4096 * 5              # working weights + codes
    m = B.gptq_workspace_min_bytes(4096, 4096, 128)
    assert 4096 * 4096 * 5 <= m < w          # the low parts of the operands are optional
    assert B.gptq_workspace_min_bytes(4096, 0, 128) == 0
    assert B.gptq_workspace_bytes(4096, 0, 128) == 0
    assert B.gptq_workspace_bytes(4096, -5, 128) == 0


def _call(lib, name, *args):
    return getattr(lib, name)(*args)


def test_invalid_arguments_rejected_on_host(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: validation fails first
    # H NULL
    assert lib.gptq_hessian_accumulate(None, fake, 16, 64, None) == 1
    # d_in not a multiple of 8
    assert lib.gptq_hessian_accumulate(fake, fake, 16, 60, None) == 1
    # negative tokens
    assert lib.gptq_hessian_accumulate(fake, fake, -1, 64, None) == 1
    # misaligned
    assert lib.gptq_hessian_accumulate(P((1 << 20) + 4), fake, 16, 64, None) == 1
    # prepare: negative damp, null outputs, missing workspace
    assert lib.gptq_prepare(fake, 64, ctypes.c_float(-1.0), 0, fake, fake, fake, 1 << 30, None) == 1
    assert lib.gptq_prepare(fake, 64, ctypes.c_float(0.01), 0, None, fake, fake, 1 << 30, None) == 1
    assert lib.gptq_prepare(fake, 64, ctypes.c_float(0.01), 0, fake, fake, None, 0, None) == 6
    assert lib.gptq_prepare(fake, 64, ctypes.c_float(0.01), 0, fake, fake, fake, 10, None) == 6
    # prepare_async: the same refusals, plus a missing or misaligned status word
    pa = lib.gptq_prepare_async
    assert pa(fake, 64, ctypes.c_float(-1.0), 0, fake, fake, fake, 1 << 30, fake, None) == 1
    assert pa(fake, 64, ctypes.c_float(0.01), 0, fake, fake, fake, 1 << 30, None, None) == 1
    assert pa(fake, 64, ctypes.c_float(0.01), 0, fake, fake, fake, 1 << 30, P((1 << 20) + 2), None) == 1
    assert pa(fake, 64, ctypes.c_float(0.01), 0, fake, fake, None, 0, fake, None) == 6

    def q(bits=4, gs=128, block=128, d_in=256, packed=None, ws=fake, ws_bytes=1 << 40):
        return lib.gptq_quantize(fake, fake, None, 64, d_in, bits, gs, block, None, fake, fake,
                                 packed, None, None, ws, ws_bytes, None)
    assert q(bits=0) == 1
    assert q(bits=9) == 1
    assert q(gs=100) == 1            # does not divide d_in
    assert q(gs=0) == 1
    assert q(block=12) == 1          # not a multiple of 8
    assert q(block=256) == 1         # above the fused kernel's width
    assert q(gs=64, block=96) == 1   # neither divides the other
    assert q(bits=5, packed=fake) == 1
    assert q(d_in=100) == 1          # not a multiple of 8
    assert q(ws=None) == 6
    assert q(ws_bytes=100) == 6
    assert lib.gptq_bf16_to_f32(None, fake, 10, None) == 1
    assert lib.gptq_hessian_accumulate_host(fake, fake, 16, 64, None, 8, None) == 1
    assert lib.gptq_hessian_accumulate_host(fake, fake, 16, 64, fake, 0, None) == 1
    assert lib.gptq_selftest_bounded_wait(0) == 1
    assert lib.gptq_selftest_bounded_wait(1 << 40) == 1
    assert lib.gptq_selftest_quotient(0, 0, fake) == 1
    assert lib.gptq_selftest_quotient(16, 0, None) == 1


def test_w4a16_arguments_rejected_on_host(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)

    def w(M=4, N=64, K=256, gs=128, path=0, X=fake, packed=fake, g_idx=None, Y=fake):
        return lib.gptq_w4a16_gemm(Y, X, packed, fake, fake, g_idx, M, N, K, gs, path, None)
    assert w(K=250) == 1             # K not a multiple of 8
    assert w(K=0) == 1
    assert w(M=-1) == 1
    assert w(gs=100) == 1            # does not divide K
    assert w(gs=0) == 1
    assert w(path=4) == 1            # no such path
    assert w(X=None) == 1
    assert w(Y=None) == 1
    assert w(X=P((1 << 20) + 2)) == 1       # X not 16-byte aligned
    assert w(packed=P((1 << 20) + 8)) == 1  # packed rows not 16-byte aligned
    # the tensor-core path refuses layouts it does not cover
    assert w(path=1, g_idx=fake) == 1       # groups given per column
    assert w(path=1, K=264, gs=-1) == 1     # K not a multiple of 32
    assert w(path=1, K=192, gs=48) == 1     # group neither divides nor is a multiple of 128
    # the decode path refuses more than 4 rows, scattered groups, groups of fewer
    # than 32 columns and K not a multiple of 32
    assert w(path=3, M=5) == 1
    assert w(path=3, g_idx=fake) == 1
    assert w(path=3, gs=16) == 1
    assert w(path=3, K=264, gs=-1) == 1
    # empty products are done without a device
    assert w(M=0) == 0
    assert w(N=0) == 0


def test_hessian_f32_arguments_rejected_on_host(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    assert B.gptq_hessian_f32_workspace_bytes(4096, 8192) >= 16 * 4096 * 4096 + 4 * 8192 * 4096
    assert B.gptq_hessian_f32_workspace_bytes(100, 16) == 0       # d_in not a multiple of 8
    assert B.gptq_hessian_f32_workspace_bytes(40000, 16) == 0     # above 32768
    assert B.gptq_hessian_f32_workspace_bytes(64, 0) == 0

    def f(n=16, d=64, chunk=8, ws=fake, ws_bytes=1 << 40, H=fake, X=fake):
        return lib.gptq_hessian_accumulate_f32(H, X, n, d, chunk, ws, ws_bytes, None)
    assert f(d=60) == 1
    assert f(chunk=0) == 1
    assert f(n=-1) == 1
    assert f(H=None) == 1
    assert f(X=P((1 << 20) + 4)) == 1     # X not 16-byte aligned
    assert f(ws=None) == 6
    assert f(ws=P((1 << 20) + 16)) == 6   # workspace not 256-byte aligned
    assert f(ws_bytes=100) == 6
    assert f(n=0) == 0                    # nothing to do, device untouched


def test_q4k_arguments_rejected_on_host(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)

    def q(d_in=512, sc6=fake, ws=fake, ws_bytes=1 << 40):
        return lib.gptq_quantize_q4k(fake, fake, None, 64, d_in, None, sc6, fake, fake, fake, fake,
                                     fake, None, None, None, ws, ws_bytes, None)
    assert q(d_in=384) == 1          # not a multiple of 256
    assert q(sc6=None) == 1
    assert q(ws=None) == 6
    assert q(ws_bytes=100) == 6


def test_a_c_program_links_and_calls_the_library(tmp_path):
    """The boundary is plain C: a C99 program includes gptq.h, links
    libgptq.so and calls the host-only entry points (no GPU needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "post_weight_quantization_accumulate_b200")
    src = tmp_path / "t.c"
    src.write_text(
        '#include <stdio.h>\n#include "gptq.h"\n'
        "int main(void) {\n"
        "  size_t ws = gptq_workspace_bytes(4096, 4096, 128);\n"
        "  size_t bad = gptq_workspace_bytes(4096, -5, 128);\n"
        '  printf("%d %zu %zu %s\\n", gptq_version(), ws, bad, gptq_status_string(1));\n'
        "  return (gptq_version() > 0 && ws > 0 && bad == 0) ? 0 : 1;\n}\n")
    exe = tmp_path / "t"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        str(src), "-L", pkg, "-lgptq", f"-Wl,-rpath,{pkg}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    version, ws, bad = r.stdout.split()[:3]
    assert int(version) == B.gptq_version() and int(ws) == B.gptq_workspace_bytes(4096, 4096, 128)
