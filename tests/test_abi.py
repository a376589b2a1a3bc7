"""The C-ABI library: loads, exports every entry point its header declares, and
validates arguments on the host (CPU only; no compute call is made)."""
import ctypes as C
import os
import re
import subprocess

import pytest

import int6_quantized_linear_b200 as ql
from int6_quantized_linear_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return ql.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(qlinear_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("qlinear_pack", "qlinear_dequant", "qlinear_gemv", "qlinear_gemm",
                     "qlinear_packed_bytes", "qlinear_status_string", "qlinear_sync_status",
                     "qlinear_gemm_workspace_bytes", "qlinear_gemv_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ql.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (qlinear_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)
    assert set(ql._SIGNATURES) == set(declared_functions())


def test_no_oracle_in_the_product():
    """The library neither defines nor links an oracle routine, and no product module imports it."""
    out = subprocess.run(["nm", "-D", ql.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert not re.search(r"\bor_(int4|int6|affine|matmul|f32|bf16)", out)
    pkg = os.path.join(ROOT, "int6_quantized_linear_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), fn
                assert "liboracle" not in src and "oracle.h" not in src, fn


@pytest.mark.parametrize("fmt,N,K,bits,group,bpw", [
    ("int4", 3, 512, 0, 0, 4.625), ("int6", 3, 512, 0, 0, 6.5625), ("int6p", 3, 512, 0, 0, 6.5625),
    ("affine", 3, 512, 2, 64, 2.5), ("affine", 3, 512, 4, 64, 4.5), ("affine", 3, 512, 8, 64, 8.5),
    ("affine", 3, 512, 4, 32, 5.0), ("affine", 3, 512, 4, 128, 4.25)])
def test_packed_bytes_closed_forms(lib, fmt, N, K, bits, group, bpw):
    c, g, s = ql.qlinear_packed_bytes(ql.Desc(fmt, N, K, bits, group))
    assert 8 * (c + g + s) == bpw * N * K


@pytest.mark.parametrize("desc", [
    ql.Desc("int4", 4, 255), ql.Desc("int4", 0, 256), ql.Desc("int6", 4, 384), ql.Desc("int6p", 4, 384),
    ql.Desc("affine", 4, 512, 3, 64), ql.Desc("affine", 4, 512, 4, 48), ql.Desc("affine", 4, 96, 2, 32)])
def test_bad_shapes_rejected(lib, desc):
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_packed_bytes(desc)
    assert e.value.status == ql.QL_ERR_SHAPE


def _call_gemv(lib, desc, codes, gmeta, steps, x, M, y, ws=0x20000, ws_bytes=1 << 24):
    d = desc.c()
    w = ql.ql_packed(codes, gmeta, steps)
    return lib.qlinear_gemv(C.byref(d), C.byref(w), x, M, y, ws, ws_bytes, None)


def test_host_validation_before_any_launch(lib):
    """Errors detected on the host come back before the library touches the device."""
    d = ql.Desc("int4", 8, 256)
    A = 0x10000  # an aligned address that is never dereferenced: validation fails first
    assert _call_gemv(lib, d, None, A, A, A, 1, A) == ql.QL_ERR_NULL
    assert _call_gemv(lib, d, A + 4, A, A, A, 1, A) == ql.QL_ERR_ALIGN
    assert _call_gemv(lib, d, A, A, A, A + 2, 1, A) == ql.QL_ERR_ALIGN
    assert _call_gemv(lib, d, A, A, A, A, 0, A) == ql.QL_ERR_RANGE
    assert _call_gemv(lib, d, A, A, A, A, 9, A) == ql.QL_ERR_RANGE
    assert _call_gemv(lib, ql.Desc("int4", 8, 100), A, A, A, A, 1, A) == ql.QL_ERR_SHAPE
    da = ql.Desc("affine", 8, 256, 4, 64)
    assert _call_gemv(lib, da, A, A, None, A, 33, A) == ql.QL_ERR_RANGE
    d6 = ql.Desc("int6", 8, 256)
    assert _call_gemv(lib, d6, A, A, A, A, 9, A) == ql.QL_ERR_RANGE  # int6 GEMV serves M <= 8
    assert _call_gemv(lib, d6, A, A, A, A, 0, A) == ql.QL_ERR_RANGE
    assert _call_gemv(lib, ql.Desc("int6", 8, 320), A, A, A, A, 1, A) == ql.QL_ERR_SHAPE  # K % 256
    assert _call_gemv(lib, d, A, A, A, A, 1, A, ws=None) == ql.QL_ERR_NULL
    assert _call_gemv(lib, d, A, A, A, A, 1, A, ws=A + 128) == ql.QL_ERR_ALIGN
    assert _call_gemv(lib, d, A, A, A, A, 1, A, ws_bytes=16) == ql.QL_ERR_SHAPE
    bad = ql.ql_desc(9, 0, 0, 0, 8, 256)
    w = ql.ql_packed(A, A, A)
    assert lib.qlinear_gemm(C.byref(bad), C.byref(w), A, 1, A, A, 1 << 20, None) == ql.QL_ERR_UNSUPPORTED
    d2 = ql.Desc("int4", 8, 256).c()
    assert lib.qlinear_gemm(C.byref(d2), C.byref(w), A, 1, A, A, 16, None) == ql.QL_ERR_SHAPE  # workspace too small
    assert lib.qlinear_gemm(C.byref(d2), C.byref(w), A, 1, A, A + 16, 1 << 20, None) == ql.QL_ERR_ALIGN
    assert ql.qlinear_gemm_workspace_bytes(ql.Desc("int4", 300, 512), 3) == 3 * 512 * 2 + 256 + 2 * 512 * 4 + (256 - 3 * 512 * 2 % 256) % 256
    for s in range(8):
        assert isinstance(ql.status_string(s), str) and ql.status_string(s)
    assert lib.qlinear_version() >= 1


def _a256(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("fmt,bits,group,N,K,M", [("int4", 0, 0, 300, 512, 1), ("int4", 0, 0, 27648, 5120, 8),
                                                  ("int6", 0, 0, 5120, 5120, 1), ("int6", 0, 0, 1000, 768, 8),
                                                  ("affine", 2, 64, 14336, 4096, 8), ("affine", 4, 128, 64, 256, 3),
                                                  ("int4", 0, 0, 131072, 16384, 1)])
def test_gemv_workspace_formula(lib, fmt, bits, group, N, K, M):
    """The GEMV workspace size is the documented sum: x words (three bytes of 24-bit fixed point per
    element, laid out for the tensor-core fragments), per-group scales and sums, the partial sums of a K
    split (for a wide layer at M=1 enough for its parts of at most 20 super-blocks), one counter per 16
    rows, a 16-byte flag record per super-block, each part rounded up to 256 bytes."""
    partial = max(4096 * 64 * M, 64 * -(-N // 64) * -(-(K // 256) // 20))  # floats
    want = (_a256(7 * M * K) + _a256(8 * M * (K // 32)) + _a256(4 * partial) + _a256(4 * ((N + 15) // 16))
            + _a256(16 * (K // 256)))
    assert ql.qlinear_gemv_workspace_bytes(ql.Desc(fmt, N, K, bits, group), M) == want


def test_gemv_workspace_covers_the_gemm_route(lib):
    """Affine calls past the multi-token range run on the GEMM: the GEMV workspace covers the GEMM's."""
    for d, M in ((ql.Desc("affine", 14336, 4096, 2, 64), 32), (ql.Desc("affine", 640, 1024, 8, 128), 8)):
        assert ql.qlinear_gemv_workspace_bytes(d, M) >= ql.qlinear_gemm_workspace_bytes(d, M)
