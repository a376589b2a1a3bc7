"""NumPy-facing wrapper over the C oracle (``oracle.c``).

Test infrastructure only: the tests, the smoke check and the benchmark's CPU
baseline call this; the product path never does.  Every function takes and
returns plain NumPy arrays with the layouts documented in ``oracle.h``.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        I64 = C.c_int64
        L.or_f32_from_f16.restype = C.c_float
        L.or_f32_from_f16.argtypes = [C.c_uint16]
        L.or_f32_from_bf16.restype = C.c_float
        L.or_f32_from_bf16.argtypes = [C.c_uint16]
        L.or_bf16_from_f32.restype = C.c_uint16
        L.or_bf16_from_f32.argtypes = [C.c_float]
        L.or_bf16_from_f64_array.argtypes = [I64, P, P]
        L.or_num_threads.restype = C.c_int
        L.or_set_num_threads.argtypes = [C.c_int]
        for name, n in (("or_int4_pack", 10), ("or_int4_unpack", 10), ("or_int4_dequant", 6),
                        ("or_int6_pack", 8), ("or_int6_unpack", 8), ("or_int6_dequant", 6),
                        ("or_int6p_pack", 8), ("or_int6p_unpack", 8), ("or_int6p_dequant", 6),
                        ("or_matmul_f64", 6)):
            getattr(L, name).argtypes = [I64, I64] + [P] * (n - 2)
        for name, n in (("or_affine_pack", 9), ("or_affine_unpack", 9), ("or_affine_dequant", 7)):
            getattr(L, name).argtypes = [I64, I64, C.c_int, C.c_int] + [P] * (n - 4)
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().or_num_threads()


def set_num_threads(n: int) -> None:
    """Thread count of the following oracle calls (for timing; results do not depend on it)."""
    lib().or_set_num_threads(int(n))


# ---- scalar conversions -------------------------------------------------------

def f32_from_f16(h: int) -> float:
    return lib().or_f32_from_f16(h)


def f32_from_bf16(b: int) -> float:
    return lib().or_f32_from_bf16(b)


def bf16_from_f32(f) -> int:
    return lib().or_bf16_from_f32(float(np.float32(f)))


def bf16_from_f64(y: np.ndarray) -> np.ndarray:
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.uint16)
    lib().or_bf16_from_f64_array(y.size, _p(y), _p(out))
    return out


# ---- int4 nested superscale ----------------------------------------------------

def int4_pack(q, sc, zc, ss, zs):
    q = _c(q, np.uint8)
    N, K = q.shape
    codes = np.empty((N, K // 2), np.uint8)
    gmeta = np.empty((N, K // 32), np.uint16)
    steps = np.empty((N, K // 256), np.uint32)
    lib().or_int4_pack(N, K, _p(q), _p(_c(sc, np.uint8)), _p(_c(zc, np.uint8)),
                       _p(_c(ss, np.uint16)), _p(_c(zs, np.uint16)),
                       _p(codes), _p(gmeta), _p(steps))
    return codes, gmeta, steps


def int4_unpack(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    q = np.empty((N, K), np.uint8)
    sc = np.empty((N, K // 32), np.uint8)
    zc = np.empty((N, K // 32), np.uint8)
    ss = np.empty((N, K // 256), np.uint16)
    zs = np.empty((N, K // 256), np.uint16)
    lib().or_int4_unpack(N, K, _p(codes), _p(_c(gmeta, np.uint16)), _p(_c(steps, np.uint32)),
                         _p(q), _p(sc), _p(zc), _p(ss), _p(zs))
    return q, sc, zc, ss, zs


def int4_dequant(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    w = np.empty((N, K), np.float32)
    lib().or_int4_dequant(N, K, _p(codes), _p(_c(gmeta, np.uint16)), _p(_c(steps, np.uint32)),
                          _p(w))
    return w


# ---- int6 symmetric ------------------------------------------------------------

def int6_pack(q, sc, st):
    q = _c(q, np.int8)
    N, K = q.shape
    codes = np.empty((N, 3 * K // 4), np.uint8)
    gmeta = np.empty((N, K // 16), np.int8)
    steps = np.empty((N, K // 256), np.uint16)
    lib().or_int6_pack(N, K, _p(q), _p(_c(sc, np.int8)), _p(_c(st, np.uint16)),
                       _p(codes), _p(gmeta), _p(steps))
    return codes, gmeta, steps


def int6_unpack(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 4 // 3
    q = np.empty((N, K), np.int8)
    sc = np.empty((N, K // 16), np.int8)
    st = np.empty((N, K // 256), np.uint16)
    lib().or_int6_unpack(N, K, _p(codes), _p(_c(gmeta, np.int8)), _p(_c(steps, np.uint16)),
                         _p(q), _p(sc), _p(st))
    return q, sc, st


def int6_dequant(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 4 // 3
    w = np.empty((N, K), np.float32)
    lib().or_int6_dequant(N, K, _p(codes), _p(_c(gmeta, np.int8)), _p(_c(steps, np.uint16)),
                          _p(w))
    return w


# ---- int6 planar (low-nibble plane + 2-bit plane per super-block) -------------

def int6p_pack(q, sc, st):
    q = _c(q, np.int8)
    N, K = q.shape
    codes = np.empty((N, 3 * K // 4), np.uint8)
    gmeta = np.empty((N, K // 16), np.int8)
    steps = np.empty((N, K // 256), np.uint16)
    lib().or_int6p_pack(N, K, _p(q), _p(_c(sc, np.int8)), _p(_c(st, np.uint16)),
                        _p(codes), _p(gmeta), _p(steps))
    return codes, gmeta, steps


def int6p_unpack(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 4 // 3
    q = np.empty((N, K), np.int8)
    sc = np.empty((N, K // 16), np.int8)
    st = np.empty((N, K // 256), np.uint16)
    lib().or_int6p_unpack(N, K, _p(codes), _p(_c(gmeta, np.int8)), _p(_c(steps, np.uint16)),
                          _p(q), _p(sc), _p(st))
    return q, sc, st


def int6p_dequant(codes, gmeta, steps):
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 4 // 3
    w = np.empty((N, K), np.float32)
    lib().or_int6p_dequant(N, K, _p(codes), _p(_c(gmeta, np.int8)), _p(_c(steps, np.uint16)),
                           _p(w))
    return w


# ---- uint32 affine -------------------------------------------------------------

def affine_pack(q, s, b, bits: int, G: int):
    q = _c(q, np.uint8)
    N, K = q.shape
    codes = np.empty((N, K * bits // 32), np.uint32)
    gmeta = np.empty((N, K // G), np.uint32)
    lib().or_affine_pack(N, K, bits, G, _p(q), _p(_c(s, np.uint16)), _p(_c(b, np.uint16)),
                         _p(codes), _p(gmeta))
    return codes, gmeta


def affine_unpack(codes, gmeta, bits: int, G: int):
    codes = _c(codes, np.uint32)
    N, K = codes.shape[0], codes.shape[1] * 32 // bits
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, K // G), np.uint16)
    b = np.empty((N, K // G), np.uint16)
    lib().or_affine_unpack(N, K, bits, G, _p(codes), _p(_c(gmeta, np.uint32)),
                           _p(q), _p(s), _p(b))
    return q, s, b


def affine_dequant(codes, gmeta, bits: int, G: int):
    codes = _c(codes, np.uint32)
    N, K = codes.shape[0], codes.shape[1] * 32 // bits
    w = np.empty((N, K), np.float32)
    lib().or_affine_dequant(N, K, bits, G, _p(codes), _p(_c(gmeta, np.uint32)), _p(w))
    return w


# ---- matmul ---------------------------------------------------------------------

def matmul_f64(x_bf16, w):
    x_bf16 = _c(x_bf16, np.uint16)
    w = _c(w, np.float32)
    M, K = x_bf16.shape
    N = w.shape[0]
    assert w.shape[1] == K
    y = np.empty((M, N), np.float64)
    lib().or_matmul_f64(M, N, K, _p(x_bf16), _p(w), _p(y))
    return y
