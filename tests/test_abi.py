"""The C-ABI library loads, exports every entry point include/sq.h declares,
and rejects bad arguments on the host without launching anything.

No GPU needed: every call here fails validation (or is the M == 0 no-op)
before the library touches the CUDA runtime, so the fake device addresses
are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from w8a8_smoothquant_int8_02_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")

A = 0x7F0000000000  # 16-byte aligned fake device address (never dereferenced)
MIS = A + 1
NUL = None


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:sq_status|const char\s*\*|int|size_t)\s+(sq_\w+)\s*\(",
                                 text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return ops.load()


def test_header_declares_the_expected_entry_points():
    assert set(declared_symbols()) == set(ops.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_exported_symbols_are_visible_to_the_dynamic_linker():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ops.library_path()],
                         capture_output=True, text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if l.strip()}
    for name in declared_symbols():
        assert name in syms, name


def test_abi_version_and_status_strings(lib):
    assert lib.sq_abi_version() == 8
    for st in range(7):
        assert ops.status_string(st).startswith("SQ_")
    assert "TIMEOUT" in ops.status_string(ops.SQ_ERR_TIMEOUT)


def c(v):
    return ctypes.c_void_p(v) if v is not None else None


def test_quantize_act_validation(lib):
    f = lib.sq_quantize_act
    ok = dict(x=A, xt=ops.SQ_BF16, M=4, K=64, s=A, qt=ops.SQ_I8, xq=A, sx=A)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["x"]), a["xt"], a["M"], a["K"], c(a["s"]), c(a.get("s_inv")), a["qt"], c(a["xq"]),
                 c(a["sx"]), a.get("flags", 0), None)

    assert call(x=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(xq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(sx=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(K=0) == ops.SQ_ERR_INVALID_ARG
    assert call(K=24) == ops.SQ_ERR_INVALID_ARG       # not a multiple of 16
    assert call(K=65536 + 16) == ops.SQ_ERR_INVALID_ARG
    assert call(M=-1) == ops.SQ_ERR_INVALID_ARG
    assert call(xt=ops.SQ_I8) == ops.SQ_ERR_INVALID_ARG
    assert call(qt=ops.SQ_BF16) == ops.SQ_ERR_INVALID_ARG
    assert call(x=MIS) == ops.SQ_ERR_MISALIGNED
    assert call(xq=A + 8) == ops.SQ_ERR_MISALIGNED
    assert call(s=A + 4) == ops.SQ_ERR_MISALIGNED
    assert call(s_inv=A + 4) == ops.SQ_ERR_MISALIGNED
    assert call(flags=2) == ops.SQ_ERR_INVALID_ARG     # unknown flag bit
    assert call(flags=0x80000001) == ops.SQ_ERR_INVALID_ARG
    assert call(M=0) == ops.SQ_OK                      # empty input: no-op
    assert call(M=0, flags=ops.SQ_OVERLAP_PREVIOUS) == ops.SQ_OK


def test_quantize_act_tensor_validation(lib):
    f = lib.sq_quantize_act_tensor
    ok = dict(x=A, xt=ops.SQ_BF16, M=4, K=64, s=A, qt=ops.SQ_E4M3, prev=A + 64, xq=A, sx=A,
              out=A + 128)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["x"]), a["xt"], a["M"], a["K"], c(a["s"]), c(a.get("s_inv")), a["qt"],
                 c(a["prev"]), c(a["xq"]), c(a["sx"]), c(a["out"]), None)

    assert call(out=NUL) == ops.SQ_ERR_INVALID_ARG     # the tensor max is required
    assert call(out=A + 64) == ops.SQ_ERR_INVALID_ARG  # aliases amax_prev
    assert call(x=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(xq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(sx=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(K=24) == ops.SQ_ERR_INVALID_ARG
    assert call(K=65536 + 16) == ops.SQ_ERR_INVALID_ARG
    assert call(M=-1) == ops.SQ_ERR_INVALID_ARG
    assert call(xt=ops.SQ_E4M3) == ops.SQ_ERR_INVALID_ARG
    assert call(qt=ops.SQ_F32) == ops.SQ_ERR_INVALID_ARG
    assert call(out=A + 130) == ops.SQ_ERR_MISALIGNED
    assert call(prev=A + 66) == ops.SQ_ERR_MISALIGNED
    assert call(x=MIS) == ops.SQ_ERR_MISALIGNED
    assert call(s=A + 4) == ops.SQ_ERR_MISALIGNED


def test_fold_smoothing_validation(lib):
    f = lib.sq_fold_smoothing
    ok = dict(p=A, pt=ops.SQ_BF16, rows=3, cols=40, s=A + 4096, axis=ops.SQ_AMAX_PER_COLUMN,
              out=A + 8192)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["p"]), a["pt"], a["rows"], a["cols"], c(a["s"]), a["axis"], c(a["out"]), None)

    assert call(p=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(s=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(out=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(out=A) == ops.SQ_ERR_INVALID_ARG          # in place is aliasing
    assert call(pt=ops.SQ_I8) == ops.SQ_ERR_INVALID_ARG
    assert call(axis=2) == ops.SQ_ERR_INVALID_ARG
    assert call(rows=-1) == ops.SQ_ERR_INVALID_ARG
    assert call(rows=2 ** 40, cols=2 ** 40) == ops.SQ_ERR_INVALID_ARG   # rows*cols overflows
    assert call(p=A + 1) == ops.SQ_ERR_MISALIGNED          # bf16 wants 2-byte alignment
    assert call(p=A + 2, pt=ops.SQ_F32) == ops.SQ_ERR_MISALIGNED
    assert call(s=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(out=A + 8194) == ops.SQ_ERR_MISALIGNED
    # empty: a no-op that accepts NULL pointers
    assert call(rows=0, p=NUL, s=NUL, out=NUL) == ops.SQ_OK
    assert call(cols=0, p=NUL, s=NUL, out=NUL) == ops.SQ_OK


def test_gemm_validation(lib):
    f = lib.sq_gemm_w8a8
    ok = dict(xq=A, sx=A, wq=A, sw=A, bias=None, M=16, N=64, K=64, y=A, yt=ops.SQ_BF16, acc=None,
              ws=None, wsn=0)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["xq"]), c(a["sx"]), c(a["wq"]), c(a["sw"]), c(a["bias"]), a["M"], a["N"],
                 a["K"], c(a["y"]), a["yt"], c(a["acc"]), c(a["ws"]), a["wsn"], None)

    assert call(xq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(wq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(y=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(N=0) == ops.SQ_ERR_INVALID_ARG
    assert call(N=12) == ops.SQ_ERR_INVALID_ARG        # not a multiple of 8
    assert call(K=40) == ops.SQ_ERR_INVALID_ARG        # not a multiple of 16
    assert call(K=133152) == ops.SQ_ERR_UNSUPPORTED    # int32 accumulator could overflow
    assert call(yt=ops.SQ_I8) == ops.SQ_ERR_INVALID_ARG
    assert call(wq=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(y=A + 8) == ops.SQ_ERR_MISALIGNED
    assert call(bias=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(sw=A + 4) == ops.SQ_ERR_MISALIGNED
    assert call(acc=A + 4) == ops.SQ_ERR_MISALIGNED
    assert call(ws=A + 16, wsn=1 << 20) == ops.SQ_ERR_MISALIGNED
    assert call(M=0) == ops.SQ_OK
    g = lib.sq_gemm_fp8
    assert g(c(A), c(A), c(A), c(A), None, 16, 64, 40, c(A), ops.SQ_BF16, None, 0, None) == ops.SQ_ERR_INVALID_ARG
    assert g(c(A), c(A), c(A), c(A), None, 0, 64, 64, c(A), ops.SQ_BF16, None, 0, None) == ops.SQ_OK


def test_gemm_noalloc_validation(lib):
    """The allocation-free GEMM rejects bad arguments on the host exactly as
    sq_gemm_w8a8 does (same checks, no launch), and M == 0 is a no-op."""
    f = lib.sq_gemm_w8a8_noalloc
    ok = dict(xq=A, sx=A, wq=A, sw=A, bias=None, M=16, N=64, K=64, y=A, yt=ops.SQ_BF16)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["xq"]), c(a["sx"]), c(a["wq"]), c(a["sw"]), c(a["bias"]), a["M"], a["N"],
                 a["K"], c(a["y"]), a["yt"], None)

    assert call(xq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(sx=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(wq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(sw=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(y=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(M=-1) == ops.SQ_ERR_INVALID_ARG
    assert call(N=0) == ops.SQ_ERR_INVALID_ARG
    assert call(N=12) == ops.SQ_ERR_INVALID_ARG        # not a multiple of 8
    assert call(K=0) == ops.SQ_ERR_INVALID_ARG
    assert call(K=40) == ops.SQ_ERR_INVALID_ARG        # not a multiple of 16
    assert call(K=133152) == ops.SQ_ERR_UNSUPPORTED    # int32 accumulator could overflow
    assert call(yt=ops.SQ_I8) == ops.SQ_ERR_INVALID_ARG
    assert call(yt=ops.SQ_E4M3) == ops.SQ_ERR_INVALID_ARG
    assert call(xq=A + 8) == ops.SQ_ERR_MISALIGNED
    assert call(wq=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(y=A + 8) == ops.SQ_ERR_MISALIGNED
    assert call(sx=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(sw=A + 4) == ops.SQ_ERR_MISALIGNED
    assert call(bias=A + 2) == ops.SQ_ERR_MISALIGNED
    assert call(M=0) == ops.SQ_OK
    assert call(M=0, xq=NUL, sx=NUL, y=NUL) == ops.SQ_OK


def test_scratch_too_small_has_its_own_message(lib):
    msg = ops.status_string(ops.SQ_ERR_SCRATCH_TOO_SMALL)
    assert msg.startswith("SQ_ERR_SCRATCH_TOO_SMALL") and "160 SMs" in msg


def test_smooth_factor_and_calibration_validation(lib):
    sf = lib.sq_smooth_factors
    assert sf(c(A), c(A), 64, 1.5, c(A), None, None) == ops.SQ_ERR_INVALID_ARG
    assert sf(c(A), c(A), 64, -0.1, c(A), None, None) == ops.SQ_ERR_INVALID_ARG
    assert sf(c(A), c(A), 64, float("nan"), c(A), None, None) == ops.SQ_ERR_INVALID_ARG
    assert sf(c(A), c(A), 0, 0.5, c(A), None, None) == ops.SQ_ERR_INVALID_ARG
    assert sf(c(A), None, 64, 0.5, c(A), None, None) == ops.SQ_ERR_INVALID_ARG
    assert sf(c(A + 2), c(A), 64, 0.5, c(A), None, None) == ops.SQ_ERR_MISALIGNED
    assert sf(c(A), c(A), 64, 0.5, c(A), c(A + 2), None) == ops.SQ_ERR_MISALIGNED
    ca = lib.sq_calibrate_amax
    assert ca(c(A), ops.SQ_BF16, 0, 64, 0, c(A), 0, None) == ops.SQ_ERR_INVALID_ARG
    assert ca(c(A), ops.SQ_BF16, 8, 60, 0, c(A), 0, None) == ops.SQ_ERR_INVALID_ARG
    assert ca(c(A), ops.SQ_BF16, 8, 64, 7, c(A), 0, None) == ops.SQ_ERR_INVALID_ARG
    assert ca(c(A), ops.SQ_E4M3, 8, 64, 0, c(A), 0, None) == ops.SQ_ERR_INVALID_ARG
    assert ca(c(MIS), ops.SQ_BF16, 8, 64, 0, c(A), 0, None) == ops.SQ_ERR_MISALIGNED
    qw = lib.sq_quantize_weight
    assert qw(c(A), ops.SQ_BF16, 64, 60, None, ops.SQ_I8, c(A), c(A), None) == ops.SQ_ERR_INVALID_ARG
    assert qw(c(A), ops.SQ_BF16, 64, 64, None, ops.SQ_I32, c(A), c(A), None) == ops.SQ_ERR_INVALID_ARG
    assert qw(c(A), ops.SQ_BF16, 64, 64, None, ops.SQ_I8, c(A), c(A + 4), None) == ops.SQ_ERR_MISALIGNED
    lin = lib.sq_linear
    assert lin(c(A), ops.SQ_BF16, None, None, c(A), c(A), None, ops.SQ_I32, 4, 64, 64, c(A), c(A),
               c(A), ops.SQ_BF16, None, 0, None) == ops.SQ_ERR_INVALID_ARG
    assert lin(c(A), ops.SQ_BF16, None, None, c(A), c(A), None, ops.SQ_I8, 0, 64, 64, c(A), c(A),
               c(A), ops.SQ_BF16, None, 0, None) == ops.SQ_OK
    assert lib.sq_probe_wait_timeout(10, None) == ops.SQ_ERR_INVALID_ARG


def test_abi_from_plain_c(tmp_path):
    """include/sq.h compiles as C11 and libsq.so links and answers from a C
    program (tests/c/abi_from_c.c): validation failures, empty no-ops and
    the version, no GPU touched."""
    import subprocess
    ops.load()  # builds libsq.so first if it is missing or stale
    lib = ops.library_path()
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), src, "-o", str(exe),
                    "-L", os.path.dirname(lib), "-l:" + os.path.basename(lib),
                    "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"


def test_rmsnorm_quantize_validation(lib):
    f = lib.sq_rmsnorm_quantize_act
    ok = dict(x=A, g=A + 0x100000, eps=1e-6, M=4, K=64, qt=ops.SQ_I8, xq=A + 0x200000,
              sx=A + 0x300000, xn=NUL)

    def call(**kw):
        a = dict(ok, **kw)
        return f(c(a["x"]), c(a["g"]), a["eps"], a["M"], a["K"], a["qt"], c(a["xq"]),
                 c(a["sx"]), c(a["xn"]), a.get("flags", 0), None)

    assert call(x=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(g=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(xq=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(sx=NUL) == ops.SQ_ERR_INVALID_ARG
    assert call(qt=ops.SQ_BF16) == ops.SQ_ERR_INVALID_ARG
    assert call(qt=ops.SQ_I4) == ops.SQ_ERR_INVALID_ARG
    assert call(K=60) == ops.SQ_ERR_INVALID_ARG             # not a multiple of 8
    assert call(K=0) == ops.SQ_ERR_INVALID_ARG
    assert call(M=-1) == ops.SQ_ERR_INVALID_ARG
    assert call(eps=0.0) == ops.SQ_ERR_INVALID_ARG
    assert call(eps=-1e-6) == ops.SQ_ERR_INVALID_ARG
    assert call(eps=float("inf")) == ops.SQ_ERR_INVALID_ARG
    assert call(eps=float("nan")) == ops.SQ_ERR_INVALID_ARG
    assert call(K=16384 + 8) == ops.SQ_ERR_UNSUPPORTED      # the row no longer fits on chip
    assert call(xq=A) == ops.SQ_ERR_INVALID_ARG             # codes over the input
    assert call(xq=A + 2 * 4 * 64 - 16) == ops.SQ_ERR_INVALID_ARG   # partial overlap
    assert call(sx=A + 0x100000 + 16) == ops.SQ_ERR_INVALID_ARG     # scales over the gain
    assert call(sx=A + 0x200000 + 64) == ops.SQ_ERR_INVALID_ARG     # scales over the codes
    assert call(x=A + 8) == ops.SQ_ERR_MISALIGNED
    assert call(g=A + 0x100000 + 4) == ops.SQ_ERR_MISALIGNED
    assert call(xq=A + 0x200000 + 8) == ops.SQ_ERR_MISALIGNED
    assert call(sx=A + 0x300000 + 2) == ops.SQ_ERR_MISALIGNED
    assert call(xn=A + 0x400000 + 4) == ops.SQ_ERR_MISALIGNED       # float4 stores
    assert call(xn=A + 256) == ops.SQ_ERR_INVALID_ARG               # the output over the input
    assert call(xn=A + 0x200000 - 512) == ops.SQ_ERR_INVALID_ARG    # ... over the codes
    assert call(xn=A + 0x300000 - 1024 + 16) == ops.SQ_ERR_INVALID_ARG   # ... over the scales
    assert call(flags=4) == ops.SQ_ERR_INVALID_ARG                   # unknown flag bit
    # empty batch: a no-op that accepts NULL pointers
    assert call(M=0, x=NUL, g=NUL, xq=NUL, sx=NUL) == ops.SQ_OK
