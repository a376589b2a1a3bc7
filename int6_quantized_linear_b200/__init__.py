"""Python binding of ``libqlinear.so``: the B200 weight-only quantized linear layer.

Argument marshalling only -- every step of the computation runs in the
library's CUDA kernels.  Functions carry the C entry points' names
(``include/qlinear.h``), take ``torch.Tensor`` arguments on a CUDA device,
pass their data pointers and the current CUDA stream, and raise
``QLinearError`` on a non-OK status.  There is no CPU fallback: if the library
is missing, the first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlinear.so")

QL_OK, QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_ALIGN, QL_ERR_RANGE, QL_ERR_UNSUPPORTED, QL_ERR_CUDA, \
    QL_ERR_TIMEOUT = range(8)
FORMATS = {"int4": 1, "int6": 2, "affine": 3, "int6p": 4}  # int6p: int6 codes in planar storage
QL_OUT_F32, QL_OUT_BF16 = 0, 1


class QLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class ql_desc(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("bits", C.c_int32), ("group", C.c_int32), ("reserved", C.c_int32),
                ("N", C.c_int64), ("K", C.c_int64)]


class ql_packed(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("gmeta", C.c_void_p), ("steps", C.c_void_p)]


ql_packed_const = ql_packed  # same layout, const in C


class ql_unpacked(C.Structure):
    _fields_ = [("q", C.c_void_p), ("meta0", C.c_void_p), ("meta1", C.c_void_p), ("step0", C.c_void_p),
                ("step1", C.c_void_p)]


ql_unpacked_out = ql_unpacked

_lib = None

# (name, argtypes) of every entry point declared in include/qlinear.h
_SIGNATURES = {
    "qlinear_version": ([], C.c_int32),
    "qlinear_status_string": ([C.c_int], C.c_char_p),
    "qlinear_packed_bytes": ([C.POINTER(ql_desc), C.POINTER(C.c_size_t), C.POINTER(C.c_size_t),
                              C.POINTER(C.c_size_t)], C.c_int),
    "qlinear_pack": ([C.POINTER(ql_desc), C.POINTER(ql_unpacked), C.POINTER(ql_packed), C.c_void_p], C.c_int),
    "qlinear_unpack": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.POINTER(ql_unpacked), C.c_void_p], C.c_int),
    "qlinear_dequant": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int32, C.c_void_p], C.c_int),
    "qlinear_gemv_workspace_bytes": ([C.POINTER(ql_desc), C.c_int64, C.POINTER(C.c_size_t)], C.c_int),
    "qlinear_gemv": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                      C.c_size_t, C.c_void_p], C.c_int),
    "qlinear_gemm_workspace_bytes": ([C.POINTER(ql_desc), C.c_int64, C.POINTER(C.c_size_t)], C.c_int),
    "qlinear_gemm": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p,
                      C.c_size_t, C.c_void_p], C.c_int),
    "qlinear_gemm_noalloc": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int64, C.c_void_p,
                              C.c_void_p], C.c_int),
    "qlinear_sync_status": ([C.c_void_p], C.c_int),
    "qlinear_set_withhold_copies": ([C.c_int32], C.c_int),
    "qlinear_gemv_bias": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int64, C.c_void_p,
                           C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p], C.c_int),
    "qlinear_gemm_bias": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.c_void_p, C.c_int64, C.c_void_p,
                           C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p], C.c_int),
    "qlinear_concat_n": ([C.POINTER(ql_desc), C.POINTER(ql_packed), C.POINTER(ql_desc), C.POINTER(ql_packed),
                          C.POINTER(ql_packed), C.c_void_p], C.c_int),
    "qlinear_quantize_meta": ([C.POINTER(ql_desc), C.c_void_p, C.c_void_p, C.POINTER(ql_unpacked), C.c_void_p],
                              C.c_int),
}


def lib():
    """Load the library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run __graft_entry__.build() or python -m int6_quantized_linear_b200._build)")
        L = C.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qlinear_status_string(status).decode()


def _check(status: int, where: str):
    if status != QL_OK:
        raise QLinearError(status, where)


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


@dataclass(frozen=True)
class Desc:
    """A quantized weight matrix's format and shape (mirrors ``ql_desc``)."""
    fmt: str
    N: int
    K: int
    bits: int = 0
    group: int = 0

    def c(self) -> ql_desc:
        return ql_desc(FORMATS[self.fmt], self.bits, self.group, 0, self.N, self.K)


def qlinear_version() -> int:
    return lib().qlinear_version()


def qlinear_packed_bytes(desc: Desc):
    c, g, s = C.c_size_t(), C.c_size_t(), C.c_size_t()
    d = desc.c()
    _check(lib().qlinear_packed_bytes(C.byref(d), C.byref(c), C.byref(g), C.byref(s)), "qlinear_packed_bytes")
    return c.value, g.value, s.value


def alloc_packed(desc: Desc, device="cuda"):
    """Allocate (uninitialised) packed buffers for ``desc`` as uint8 tensors."""
    import torch
    c, g, s = qlinear_packed_bytes(desc)
    return (torch.empty(c, dtype=torch.uint8, device=device), torch.empty(g, dtype=torch.uint8, device=device),
            torch.empty(max(s, 16), dtype=torch.uint8, device=device))


def qlinear_pack(desc: Desc, q, meta0, meta1, step0, step1, codes, gmeta, steps, stream=None):
    d = desc.c()
    u = ql_unpacked(_ptr(q), _ptr(meta0), _ptr(meta1), _ptr(step0), _ptr(step1))
    o = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_pack(C.byref(d), C.byref(u), C.byref(o), _stream(stream)), "qlinear_pack")


def qlinear_unpack(desc: Desc, codes, gmeta, steps, q, meta0=None, meta1=None, step0=None, step1=None,
                   stream=None):
    d = desc.c()
    i = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    o = ql_unpacked(_ptr(q), _ptr(meta0), _ptr(meta1), _ptr(step0), _ptr(step1))
    _check(lib().qlinear_unpack(C.byref(d), C.byref(i), C.byref(o), _stream(stream)), "qlinear_unpack")


def qlinear_dequant(desc: Desc, codes, gmeta, steps, out, out_dtype: int, stream=None):
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_dequant(C.byref(d), C.byref(w), _ptr(out), out_dtype, _stream(stream)),
           "qlinear_dequant")


def qlinear_quantize_meta(desc: Desc, scale, zero, meta0, meta1, step0, step1, stream=None):
    """Float per-group metadata (float32 CUDA tensors) -> codes and fp16 step bits in the given
    output tensors (int4: sc, zc u8 [N][K/32], ss, zs [N][K/256] 16-bit; int6: sc i8 [N][K/16],
    st [N][K/256]; pass None for the unused ones).  Out-of-domain inputs show up as QL_ERR_RANGE
    from qlinear_sync_status()."""
    d = desc.c()
    o = ql_unpacked(None, _ptr(meta0), _ptr(meta1), _ptr(step0), _ptr(step1))
    _check(lib().qlinear_quantize_meta(C.byref(d), _ptr(scale), _ptr(zero), C.byref(o), _stream(stream)),
           "qlinear_quantize_meta")


def qlinear_gemv_workspace_bytes(desc: Desc, M: int) -> int:
    d = desc.c()
    n = C.c_size_t()
    _check(lib().qlinear_gemv_workspace_bytes(C.byref(d), M, C.byref(n)), "qlinear_gemv_workspace_bytes")
    return n.value


def alloc_gemv_workspace(desc: Desc, M: int, device="cuda"):
    import torch
    return torch.empty(qlinear_gemv_workspace_bytes(desc, M), dtype=torch.uint8, device=device)


def qlinear_gemv(desc: Desc, codes, gmeta, steps, x, M: int, y, workspace=None, stream=None):
    """``workspace``: a uint8 CUDA tensor of at least qlinear_gemv_workspace_bytes(desc, M) bytes;
    allocated here when omitted."""
    if workspace is None:
        workspace = alloc_gemv_workspace(desc, M, x.device)
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_gemv(C.byref(d), C.byref(w), _ptr(x), M, _ptr(y), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)), "qlinear_gemv")


def qlinear_gemv_bias(desc: Desc, codes, gmeta, steps, x, M: int, bias, y, workspace=None, stream=None):
    """qlinear_gemv with a bf16 [N] bias added before the rounding to bf16."""
    if workspace is None:
        workspace = alloc_gemv_workspace(desc, M, x.device)
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_gemv_bias(C.byref(d), C.byref(w), _ptr(x), M, _ptr(bias), _ptr(y), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "qlinear_gemv_bias")


def qlinear_concat_n(desc_a: Desc, packed_a, desc_b: Desc, packed_b, out, stream=None):
    """Stack two packed layers along N into ``out`` = (codes, gmeta, steps) of the stacked layer."""
    da, db = desc_a.c(), desc_b.c()
    wa = ql_packed(*[_ptr(t) for t in packed_a])
    wb = ql_packed(*[_ptr(t) for t in packed_b])
    o = ql_packed(*[_ptr(t) for t in out])
    _check(lib().qlinear_concat_n(C.byref(da), C.byref(wa), C.byref(db), C.byref(wb), C.byref(o), _stream(stream)),
           "qlinear_concat_n")


def qlinear_gemm_workspace_bytes(desc: Desc, M: int) -> int:
    d = desc.c()
    n = C.c_size_t()
    _check(lib().qlinear_gemm_workspace_bytes(C.byref(d), M, C.byref(n)), "qlinear_gemm_workspace_bytes")
    return n.value


def alloc_gemm_workspace(desc: Desc, M: int, device="cuda"):
    """Allocate a workspace for qlinear_gemm (torch allocations are 256-byte aligned)."""
    import torch
    return torch.empty(qlinear_gemm_workspace_bytes(desc, M), dtype=torch.uint8, device=device)


def qlinear_gemm(desc: Desc, codes, gmeta, steps, x, M: int, y, workspace=None, stream=None):
    """``workspace``: a uint8 CUDA tensor of at least qlinear_gemm_workspace_bytes(desc, M) bytes;
    allocated here when omitted."""
    if workspace is None:
        workspace = alloc_gemm_workspace(desc, M, x.device)
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_gemm(C.byref(d), C.byref(w), _ptr(x), M, _ptr(y), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)), "qlinear_gemm")


def qlinear_gemm_bias(desc: Desc, codes, gmeta, steps, x, M: int, bias, y, workspace=None, stream=None):
    """qlinear_gemm with a bf16 [N] bias added before the rounding to bf16."""
    if workspace is None:
        workspace = alloc_gemm_workspace(desc, M, x.device)
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_gemm_bias(C.byref(d), C.byref(w), _ptr(x), M, _ptr(bias), _ptr(y), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "qlinear_gemm_bias")


def qlinear_gemm_noalloc(desc: Desc, codes, gmeta, steps, x, M: int, y, stream=None):
    """qlinear_gemm without a workspace argument, for callers that may not allocate device memory:
    the library uses its own fixed 32 MiB device array (shared by every call on the device, so calls
    must not overlap on the GPU).  Raises QLinearError(QL_ERR_RANGE) when the problem needs more."""
    d = desc.c()
    w = ql_packed(_ptr(codes), _ptr(gmeta), _ptr(steps))
    _check(lib().qlinear_gemm_noalloc(C.byref(d), C.byref(w), _ptr(x), M, _ptr(y), _stream(stream)),
           "qlinear_gemm_noalloc")


def qlinear_set_withhold_copies(on: bool) -> None:
    """Whether the current device's kernels start no copies, so that their first wait for data runs
    out (after about 1 s).  For tests of the give-up path (QL_ERR_TIMEOUT)."""
    _check(lib().qlinear_set_withhold_copies(1 if on else 0), "qlinear_set_withhold_copies")


def qlinear_sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status (QL_OK / QL_ERR_TIMEOUT / ...)."""
    return lib().qlinear_sync_status(_stream(stream))
