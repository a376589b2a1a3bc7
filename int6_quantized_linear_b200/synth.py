"""Seeded synthetic inputs for the quantized linear layer.

Random draws only -- no packing, dequantisation or matmul arithmetic lives
here -- so the CUDA path and the CPU oracle can both be fed from this module
without sharing any of the method's code.

Recipe (one ``numpy.random.SeedSequence(seed)`` spawns four child streams,
drawn in this order: codes, group codes, steps, activations):

* int4 nested superscale: codes uniform 0..15; per-group (32) uint8 scale and
  zero codes uniform 0..255; per-256 fp16 scale step uniform in
  [2^-14, 2^-10]; per-256 fp16 zero step uniform in [2^-6, 2^-5].
* int6 symmetric: codes uniform -32..31; per-group (16) int8 scale code
  uniform in -127..127 without 0; per-256 fp16 step uniform in [2^-14, 2^-10].
* uint32 affine: codes uniform 0..2^bits-1; per-group bf16 scale uniform in
  [1e-3, 1e-2]; per-group bf16 bias uniform in [-0.1, 0.1].
* activations: bf16 (nearest-even) of float32 standard normal draws.

fp16 values are produced by NumPy's float64 -> float16 cast (nearest-even);
bf16 values by nearest-even rounding of float32 draws.  All 16-bit floats are
returned as raw uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def _streams(seed: int, n: int = 4):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def _bf16_bits(a32: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(a32, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _f16_bits(a64: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a64.astype(np.float16)).view(np.uint16)


def int4_weights(seed: int, N: int, K: int) -> dict:
    assert K % 256 == 0
    rc, rg, rs, _ = _streams(seed)
    q = rc.integers(0, 16, size=(N, K), dtype=np.uint8)
    sc = rg.integers(0, 256, size=(N, K // 32), dtype=np.uint8)
    zc = rg.integers(0, 256, size=(N, K // 32), dtype=np.uint8)
    ss = _f16_bits(rs.uniform(2.0 ** -14, 2.0 ** -10, size=(N, K // 256)))
    zs = _f16_bits(rs.uniform(2.0 ** -6, 2.0 ** -5, size=(N, K // 256)))
    return dict(q=q, sc=sc, zc=zc, ss=ss, zs=zs)


def int6_weights(seed: int, N: int, K: int) -> dict:
    assert K % 256 == 0
    rc, rg, rs, _ = _streams(seed)
    q = rc.integers(-32, 32, size=(N, K), dtype=np.int8)
    c = rg.integers(-127, 127, size=(N, K // 16), dtype=np.int16)  # -127..126
    sc = np.where(c >= 0, c + 1, c).astype(np.int8)                  # -127..-1, 1..127
    st = _f16_bits(rs.uniform(2.0 ** -14, 2.0 ** -10, size=(N, K // 256)))
    return dict(q=q, sc=sc, st=st)


def affine_weights(seed: int, N: int, K: int, bits: int, G: int) -> dict:
    assert bits in (2, 4, 8) and K % G == 0
    rc, rg, _, _ = _streams(seed)
    q = rc.integers(0, 1 << bits, size=(N, K), dtype=np.uint8)
    s = _bf16_bits(rg.uniform(1e-3, 1e-2, size=(N, K // G)).astype(np.float32))
    b = _bf16_bits(rg.uniform(-0.1, 0.1, size=(N, K // G)).astype(np.float32))
    return dict(q=q, s=s, b=b)


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """bf16 bit patterns [M][K]; rows 0..M-1 are the first rows of any larger draw."""
    _, _, _, rx = _streams(seed)
    return _bf16_bits(rx.standard_normal(size=(M, K), dtype=np.float32))


@dataclass(frozen=True)
class Workload:
    """One synthetic layer: format, shape, batch sizes and seed."""
    name: str
    fmt: str            # "int4" | "int6" | "int6p" (int6 codes, planar storage) | "affine"
    N: int
    K: int
    Ms: tuple
    seed: int
    bits: int = 0
    group: int = 0

    def weights(self, N: int | None = None) -> dict:
        n = self.N if N is None else N
        if self.fmt == "int4":
            return int4_weights(self.seed, n, self.K)
        if self.fmt in ("int6", "int6p"):
            return int6_weights(self.seed, n, self.K)
        return affine_weights(self.seed, n, self.K, self.bits, self.group)

    def x(self, M: int) -> np.ndarray:
        return activations(self.seed, M, self.K)

    def desc_args(self) -> dict:
        return dict(fmt=self.fmt, N=self.N, K=self.K, bits=self.bits, group=self.group)


# The layer shapes the library is measured and checked on.
WORKLOADS = {
    "int4_gemv_2048x2048": Workload("int4_gemv_2048x2048", "int4", 2048, 2048, (1,), 0),
    "int4_gemv_k5120_n27648": Workload("int4_gemv_k5120_n27648", "int4", 27648, 5120, (1, 4, 8), 1),
    "int4_gemv_k27648_n5120": Workload("int4_gemv_k27648_n5120", "int4", 5120, 27648, (1, 4, 8), 1),
    "int6_gemv_k5120_n5120": Workload("int6_gemv_k5120_n5120", "int6", 5120, 5120, (1, 4), 2),
    "int6_gemv_k5120_n27648": Workload("int6_gemv_k5120_n27648", "int6", 27648, 5120, (1, 4), 2),
    # the same int6 layers with their codes in planar storage (a 4-bit and a 2-bit plane)
    "int6p_gemv_k5120_n5120": Workload("int6p_gemv_k5120_n5120", "int6p", 5120, 5120, (1, 4), 2),
    "int6p_gemv_k5120_n27648": Workload("int6p_gemv_k5120_n27648", "int6p", 27648, 5120, (1, 4), 2),
    "int4_gemm_k5120_n27648": Workload("int4_gemm_k5120_n27648", "int4", 27648, 5120,
                                       (512, 2048, 8192), 3),
    "affine2_k4096_n14336": Workload("affine2_k4096_n14336", "affine", 14336, 4096, (1, 32), 4, 2, 64),
    "affine4_k4096_n14336": Workload("affine4_k4096_n14336", "affine", 14336, 4096, (1, 32), 4, 4, 64),
    "affine8_k4096_n14336": Workload("affine8_k4096_n14336", "affine", 14336, 4096, (1, 32), 4, 8, 64),
}
