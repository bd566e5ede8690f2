"""The C ABI without a GPU: the library loads, exports every function that
include/fa.h declares, names every status, and rejects bad arguments with the
documented status before any CUDA call (no pointer is dereferenced; the fake
device addresses below are never touched).  The header is plain C99, and a C
program linked against the library calls it."""
import ctypes
import os
import re

import pytest

import flash_fwd_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE = 0, 1, 2, 3, 4
A = ctypes.c_void_p(0x10000)       # 16-byte aligned fake address
M = ctypes.c_void_p(0x10001)       # misaligned
NULL = ctypes.c_void_p(0)
S = ctypes.c_void_p(0)             # stream


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_function():
    lib = fa.load_library()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in fa.h but not exported"


def declared_arity():
    """{function: number of parameters} from the declarations in fa.h."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_argument_counts_match_the_header():
    lib = fa.load_library()
    arity = declared_arity()
    assert set(arity) == set(declared_functions())
    for name, n in arity.items():
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, f"{name}: the binding sets no argtypes"
        assert len(argtypes) == n, f"{name}: header has {n} parameters, binding {len(argtypes)}"


def test_status_strings():
    for code in range(0, 8):
        assert isinstance(fa.fa_status_string(code), str) and fa.fa_status_string(code)
    assert fa.fa_status_string(0) == "ok"
    assert fa.fa_status_string(999) == "unknown status"


def _fwd(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, scale=0.125, causal=0, dtype=1):
    return fa.load_library().fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, S)


@pytest.mark.parametrize("kw,expect", [
    (dict(d=96), UNSUPPORTED),
    (dict(d=32), UNSUPPORTED),
    (dict(d=512), UNSUPPORTED),
    (dict(B=0), INVALID),
    (dict(H=-1), INVALID),
    (dict(N=0), INVALID),
    (dict(dtype=7), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(scale=0.0), INVALID),
    (dict(scale=-0.125), INVALID),
    (dict(q=NULL), INVALID),
    (dict(lse=NULL), INVALID),
    (dict(k=M), MISALIGNED),
    (dict(o=M), MISALIGNED),
    (dict(B=1 << 20, H=1 << 10, N=512), UNSUPPORTED),   # more CTAs than a one-dimensional grid holds
])
def test_fwd_rejects(kw, expect):
    assert _fwd(**kw) == expect


def test_fwd_blocksparse_requires_mask():
    lib = fa.load_library()
    assert lib.fa_fwd_blocksparse(A, A, A, A, A, NULL, 1, 1, 128, 64, 0.1, 0, 1, S) == INVALID


def test_workspace_bytes():
    lib = fa.load_library()
    B, H, N, d = 2, 3, 1000, 128
    got = lib.fa_bwd_workspace_bytes(B, H, N, d)
    npad = (N + 127) // 128 * 128          # per-row statistics padded to whole 128-row blocks
    assert got == 2 * B * H * npad * 4 + B * H * N * d * 4
    assert lib.fa_bwd_workspace_bytes(0, 1, 1, 64) == 0
    assert lib.fa_bwd_workspace_bytes(1, 1, 1, 96) == 0


def _bwd(ws=A, ws_bytes=None, d=64, N=128, dq=A, mask=None):
    lib = fa.load_library()
    if ws_bytes is None:
        ws_bytes = lib.fa_bwd_workspace_bytes(1, 1, N, d)
    args = [A, A, A, A, A, A, dq, A, A, ws, ws_bytes]
    tail = [1, 1, N, d, 0.125, 0, 1, S]
    if mask is None:
        return lib.fa_bwd(*args, *tail)
    return lib.fa_bwd_blocksparse(*args, mask, *tail)


def test_bwd_rejects():
    lib = fa.load_library()
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 64)
    assert _bwd(ws=NULL) == WORKSPACE
    assert _bwd(ws_bytes=need - 1) == WORKSPACE
    assert _bwd(ws=M) == MISALIGNED
    assert _bwd(dq=NULL) == INVALID
    assert _bwd(dq=M) == MISALIGNED
    assert _bwd(d=80) == UNSUPPORTED
    assert _bwd(mask=NULL) == INVALID


def test_deterministic_workspace_and_rejects():
    lib = fa.load_library()
    B, H, Nq, Nk, d = 2, 3, 1000, 700, 256
    npad = (Nq + 127) // 128 * 128          # two per-row statistics, no dQ accumulator
    assert lib.fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, d) == 2 * B * H * npad * 4
    assert lib.fa_bwd_deterministic_workspace_bytes(1, 1, 1, 0, 64) == 0
    assert lib.fa_bwd_deterministic_workspace_bytes(1, 1, 1, 1, 96) == 0
    need = lib.fa_bwd_deterministic_workspace_bytes(1, 1, 128, 128, 64)

    def det(ws=A, ws_bytes=need, d=64, dq=A, scale=0.125):
        return lib.fa_bwd_deterministic(A, A, A, A, A, A, dq, A, A, ws, ws_bytes, 1, 1, 128, 128, d, scale, 0,
                                        -1, -1, NULL, NULL, 1, S)
    assert det(ws=NULL) == WORKSPACE
    assert det(ws_bytes=need - 1) == WORKSPACE
    assert det(ws=M) == MISALIGNED
    assert det(dq=NULL) == INVALID
    assert det(d=80) == UNSUPPORTED
    assert det(scale=0.0) == INVALID


def test_fp8_entry_points_reject():
    lib = fa.load_library()
    F = A   # 16-byte aligned fake device address (no launch happens on these paths)

    def quant(d=128, dtype=1, q=A, sq=F, signs=NULL):
        return lib.fa_fp8_quantize_qkv(q, A, A, A, A, A, sq, F, F, 1, 1, 128, d, signs, dtype, S)

    def fwd8(d=128, out_dtype=1, o=A, scale=0.1, sq=F):
        return lib.fa_fwd_fp8(A, A, A, sq, F, F, o, A, 1, 1, 128, d, ctypes.c_float(scale), 0, out_dtype, S)
    assert quant(q=NULL) == INVALID
    assert quant(d=96) == UNSUPPORTED
    assert quant(dtype=7) == INVALID
    assert quant(q=M) == MISALIGNED
    assert quant(sq=ctypes.c_void_p(0x10002)) == MISALIGNED
    assert fwd8(d=96) == UNSUPPORTED          # the FP8 forward is built for d = 64, 128 and 256
    assert fwd8(out_dtype=7) == INVALID
    assert fwd8(o=M) == MISALIGNED
    assert fwd8(scale=-1.0) == INVALID
    assert fwd8(sq=NULL) == INVALID


def test_profile_read_rejects_null():
    lib = fa.load_library()
    assert lib.fa_profile_read(None, None) == INVALID
    assert lib.fa_version() >= 100


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "fa.h"

int main(void) {
    /* calls that need no GPU: the version, a status name, a workspace size,
       and an argument check that returns before any CUDA call */
    int rc = fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 64, 0.125f, 0, FA_BF16, NULL);
    size_t ws = fa_bwd_workspace_bytes(1, 1, 128, 64);
    printf("%d %d %s %zu\n", fa_version(), rc, fa_status_string(FA_ERR_WORKSPACE), ws);
    return 0;
}
"""


def test_header_is_plain_c_and_callable_from_c(tmp_path):
    # the boundary is a C ABI: the header compiles as C99, and a C program
    # linked against the library calls it
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(fa.library_path())
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lfa_b200",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    version, rc, *rest = out.stdout.split()
    assert int(version) == fa.load_library().fa_version()
    assert int(rc) == INVALID
    assert int(rest[-1]) == fa.fa_bwd_workspace_bytes(1, 1, 128, 64) > 0
    assert " ".join(rest[:-1]) == fa.fa_status_string(WORKSPACE)


def test_every_entry_point_is_documented():
    # a comment directly above each declaration, or the function named in a comment block
    src = open(HEADER).read()
    comments = " ".join(re.findall(r"/\*.*?\*/", src, flags=re.S))
    lines = src.split("\n")
    for i, line in enumerate(lines):
        m = re.match(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", line)
        if m:
            above = "\n".join(lines[max(0, i - 3):i])
            assert "*/" in above or m.group(1) in comments, m.group(1)

