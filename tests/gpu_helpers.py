"""Helpers for the GPU parity tests: build a quantized layer on the device from
seeded synthetic inputs, and compute the oracle's answer for chosen rows.

The CUDA side is reached only through the C-ABI binding; the expected values
come only from the CPU oracle, fed with the same seeded inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import int6_quantized_linear_b200 as ql
from int6_quantized_linear_b200 import synth
from oracle import oracle_c as OC


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor, dtype) -> np.ndarray:
    return t.cpu().numpy().view(dtype)


class Layer:
    """One quantized weight matrix, packed on the GPU by qlinear_pack."""

    def __init__(self, fmt: str, N: int, K: int, seed: int, bits: int = 0, group: int = 0, weights=None):
        self.fmt, self.N, self.K, self.bits, self.group = fmt, N, K, bits, group
        self.desc = ql.Desc(fmt, N, K, bits, group)
        if weights is None:
            if fmt == "int4":
                weights = synth.int4_weights(seed, N, K)
            elif fmt in ("int6", "int6p"):
                weights = synth.int6_weights(seed, N, K)
            else:
                weights = synth.affine_weights(seed, N, K, bits, group)
        self.w = weights
        self.codes, self.gmeta, self.steps = ql.alloc_packed(self.desc)
        u = self.unpacked_host()
        du = [dev(a) if a is not None else None for a in u]
        ql.qlinear_pack(self.desc, *du, self.codes, self.gmeta, self.steps)
        torch.cuda.synchronize()

    def unpacked_host(self):
        w = self.w
        if self.fmt == "int4":
            return w["q"], w["sc"], w["zc"], w["ss"], w["zs"]
        if self.fmt in ("int6", "int6p"):
            return w["q"], w["sc"], None, w["st"], None
        return w["q"], w["s"], w["b"], None, None

    def packed(self):
        return self.codes, self.gmeta, self.steps

    # ---- oracle side ----
    def oracle_pack(self, rows=None):
        sel = (lambda a: a) if rows is None else (lambda a: a[rows])
        w = self.w
        if self.fmt == "int4":
            return OC.int4_pack(sel(w["q"]), sel(w["sc"]), sel(w["zc"]), sel(w["ss"]), sel(w["zs"]))
        if self.fmt == "int6":
            return OC.int6_pack(sel(w["q"]), sel(w["sc"]), sel(w["st"]))
        if self.fmt == "int6p":
            return OC.int6p_pack(sel(w["q"]), sel(w["sc"]), sel(w["st"]))
        return OC.affine_pack(sel(w["q"]), sel(w["s"]), sel(w["b"]), self.bits, self.group)

    def oracle_w(self, rows=None) -> np.ndarray:
        p = self.oracle_pack(rows)
        if self.fmt == "int4":
            return OC.int4_dequant(*p)
        if self.fmt == "int6":
            return OC.int6_dequant(*p)
        if self.fmt == "int6p":
            return OC.int6p_dequant(*p)
        return OC.affine_dequant(*p, self.bits, self.group)

    def packed_host(self):
        c, g, s = self.packed()
        gt = {"int4": np.uint16, "int6": np.int8, "int6p": np.int8, "affine": np.uint32}[self.fmt]
        st = {"int4": np.uint32, "int6": np.uint16, "int6p": np.uint16, "affine": np.uint8}[self.fmt]
        ct = np.uint32 if self.fmt == "affine" else np.uint8
        nc, ng, ns = ql.qlinear_packed_bytes(self.desc)
        return (host(c, np.uint8)[:nc].view(ct).reshape(self.N, -1),
                host(g, np.uint8)[:ng].view(gt).reshape(self.N, -1),
                host(s, np.uint8)[:ns].view(st).reshape(self.N, -1) if ns else None)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def assert_close(y_bits: np.ndarray, y_ref: np.ndarray, what: str = "", rms: float | None = None):
    """Gate: |y - y_ref| <= 1e-2 * rms(y_ref) + 1e-3 + half a bf16 ulp of y_ref, elementwise.

    The last term admits the one unavoidable rounding of the result to bf16; the
    first two are the stated fp32-accumulation budget."""
    y = bf16_to_f64(y_bits)
    if rms is None:
        rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(y - y_ref)
    tol = 1e-2 * rms + 1e-3 + half_ulp_bf16(y_ref)
    bad = err > tol
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst excess "
                           f"{float(np.max(err - tol)):.3e}, rms {rms:.3e}")
    return float(np.max(np.maximum(err - half_ulp_bf16(y_ref), 0)) / max(rms, 1e-30))


def x_dev(K: int, M: int, seed: int):
    xb = synth.activations(seed, M, K)
    return xb, dev(xb)


def run_gemv(layer: Layer, xd: torch.Tensor, M: int) -> np.ndarray:
    y = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_gemv(layer.desc, *layer.packed(), xd, M, y)
    assert ql.qlinear_sync_status() == ql.QL_OK
    return host(y.view(torch.int16), np.uint16)


def run_gemm(layer: Layer, xd: torch.Tensor, M: int) -> np.ndarray:
    y = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_gemm(layer.desc, *layer.packed(), xd, M, y)
    assert ql.qlinear_sync_status() == ql.QL_OK
    return host(y.view(torch.int16), np.uint16)
