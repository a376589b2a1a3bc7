"""Hand-built inputs at the edges of the method, for the edge-case parity tests.

Random draws and bit patterns only -- no packing, dequantisation or matmul
arithmetic lives here -- so the CUDA path and the CPU oracle can both be fed
from this module.  Every weight builder returns the unpacked fields that
``qlinear_pack`` and the oracle take, plus one category label per weight row;
the parity tests gate each (row category, activation kind) block on its own
rms, so a failure names the case.

Weight rows cycle through these categories (row n has category n % 6):

int4 (ExecuTorch PR "[cuda] Nestest Superscale Quantization for CUDA Weights
(int4 / int6)", "Quant schema update": w = (q - zc*zs) * (sc*ss)):
  0 synthetic   the workload recipe's ranges
  1 extremes    scale and zero codes 0 or 255, codes mostly 0 or 15
  2 subnormal   fp16 scale and zero steps subnormal (exponent field 0)
  3 zero steps  per super-block the scale step, the zero step or both +-0
  4 zero slots  zero step 1/16 and zero code 16*z, code z at every k with
                k % 16 == OUT_SLOT, so those weights are exactly 0
  5 large/neg   steps of either sign with magnitudes in [1, 256]
int6 (same section: w = q * (sc*st)):
  0 synthetic, 1 extremes (scale codes -128, -127, 127; codes -32 or 31),
  2 subnormal steps, 3 zero steps and zero scale codes, 4 zero slots (code 0
  at k % 16 == OUT_SLOT), 5 steps of either sign in [1, 4096]
affine (Transformers "Metal" quantization page: w = q * scale + bias):
  0 synthetic, 1 scale 0 (bias only), 2 negative scales and biases of larger
  magnitude, 3 subnormal bf16 scale and bias, 4 zero slots (bias 0, code 0
  at k % 16 == OUT_SLOT), 5 scale and bias of either sign in [2^8, 2^16]

Activation kinds (bf16 bit patterns, one row each):
  normal     N(0, 1)
  outlier10  N(0, 1), and at every k % 16 == OUT_SLOT an element 2^10 times
             the largest magnitude of the other 15 elements of its 16-block
  outlier7   the same with 2^7
  subnormal  every element a bf16 subnormal (exponent field 0) of random sign
  zero_grp   N(0, 1) with a random half of the 32-element groups all zero
  mixed_sub  N(0, 1) with every fourth element replaced by a subnormal
  wide20     N(0, 1) with the OUT_SLOT elements at +-2^20 (a row range of
             about 2^20 .. 2^30: inside the GEMM's exact fp16 range)
"""
from __future__ import annotations

import numpy as np

OUT_SLOT = 5           # k % 16 of the planted outliers and zero weights
N_CATS = 6
INT4_CATS = ("synthetic", "extremes", "subnormal", "zero steps", "zero slots", "large/neg")
INT6_CATS = ("synthetic", "extremes", "subnormal", "zero steps", "zero slots", "large/neg")
AFFINE_CATS = ("synthetic", "scale 0", "negative", "subnormal", "zero slots", "large")
X_KINDS = ("normal", "outlier10", "outlier7", "subnormal", "zero_grp", "mixed_sub", "wide20")


def _rng(seed: int, salt: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, salt]))


def _f16(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, np.float64).astype(np.float16)).view(np.uint16)


def _bf16(a) -> np.ndarray:
    """Nearest-even bf16 bit patterns of float32 values."""
    u = np.ascontiguousarray(np.asarray(a, np.float32)).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _signs(r, shape) -> np.ndarray:
    return np.where(r.integers(0, 2, size=shape) == 1, -1.0, 1.0)


def categories(N: int) -> np.ndarray:
    return np.arange(N) % N_CATS


def _slot_mask(K: int) -> np.ndarray:
    return (np.arange(K) % 16) == OUT_SLOT


def int4_edge(N: int, K: int, seed: int) -> dict:
    assert K % 256 == 0
    r = _rng(seed, 4)
    cat = categories(N)
    q = r.integers(0, 16, size=(N, K), dtype=np.uint8)
    sc = r.integers(0, 256, size=(N, K // 32), dtype=np.uint8)
    zc = r.integers(0, 256, size=(N, K // 32), dtype=np.uint8)
    ss = _f16(r.uniform(2.0 ** -14, 2.0 ** -10, size=(N, K // 256)))
    zs = _f16(r.uniform(2.0 ** -6, 2.0 ** -5, size=(N, K // 256)))
    c = cat == 1
    sc[c] = np.where(r.integers(0, 2, size=sc[c].shape) == 1, 255, 0).astype(np.uint8)
    zc[c] = np.where(r.integers(0, 2, size=zc[c].shape) == 1, 255, 0).astype(np.uint8)
    q[c] = np.where(r.integers(0, 4, size=q[c].shape) == 0, q[c],
                    np.where(r.integers(0, 2, size=q[c].shape) == 1, 15, 0)).astype(np.uint8)
    c = cat == 2
    ss[c] = r.integers(1, 0x400, size=ss[c].shape).astype(np.uint16)
    zs[c] = r.integers(1, 0x400, size=zs[c].shape).astype(np.uint16)
    c = cat == 3
    pick = r.integers(0, 4, size=ss[c].shape)  # 0: scale step 0, 1: zero step 0, 2: both -0, 3: neither
    ss[c] = np.where(pick == 0, 0, np.where(pick == 2, 0x8000, ss[c])).astype(np.uint16)
    zs[c] = np.where(pick == 1, 0, np.where(pick == 2, 0x8000, zs[c])).astype(np.uint16)
    c = cat == 4
    z = r.integers(0, 16, size=(int(c.sum()), K // 32))
    zs[c] = 0x2C00                                       # fp16 1/16
    zc[c] = (16 * z).astype(np.uint8)                    # zero = z exactly
    qz = q[c]
    qz[:, _slot_mask(K)] = np.repeat(z, 32, axis=1)[:, _slot_mask(K)].astype(np.uint8)
    q[c] = qz
    c = cat == 5
    ss[c] = _f16(_signs(r, ss[c].shape) * r.uniform(1.0, 256.0, size=ss[c].shape))
    zs[c] = _f16(_signs(r, zs[c].shape) * r.uniform(1.0, 256.0, size=zs[c].shape))
    return dict(q=q, sc=sc, zc=zc, ss=ss, zs=zs, cat=cat)


def int6_edge(N: int, K: int, seed: int) -> dict:
    assert K % 256 == 0
    r = _rng(seed, 6)
    cat = categories(N)
    q = r.integers(-32, 32, size=(N, K), dtype=np.int8)
    sc = r.integers(-128, 128, size=(N, K // 16)).astype(np.int8)
    st = _f16(r.uniform(2.0 ** -14, 2.0 ** -10, size=(N, K // 256)))
    c = cat == 1
    sc[c] = np.array([-128, -127, 127], np.int8)[r.integers(0, 3, size=sc[c].shape)]
    q[c] = np.where(r.integers(0, 4, size=q[c].shape) == 0, q[c],
                    np.where(r.integers(0, 2, size=q[c].shape) == 1, 31, -32)).astype(np.int8)
    c = cat == 2
    st[c] = (r.integers(1, 0x400, size=st[c].shape) | (r.integers(0, 2, size=st[c].shape) << 15)).astype(np.uint16)
    c = cat == 3
    st[c] = np.where(r.integers(0, 3, size=st[c].shape) == 0, 0, st[c]).astype(np.uint16)
    sc[c] = np.where(r.integers(0, 3, size=sc[c].shape) == 0, 0, sc[c]).astype(np.int8)
    c = cat == 4
    qz = q[c]
    qz[:, _slot_mask(K)] = 0
    q[c] = qz
    c = cat == 5
    st[c] = _f16(_signs(r, st[c].shape) * r.uniform(1.0, 4096.0, size=st[c].shape))
    return dict(q=q, sc=sc, st=st, cat=cat)


def affine_edge(N: int, K: int, bits: int, G: int, seed: int) -> dict:
    assert K % G == 0
    r = _rng(seed, 8 + bits)
    cat = categories(N)
    q = r.integers(0, 1 << bits, size=(N, K), dtype=np.uint8)
    s = r.uniform(1e-3, 1e-2, size=(N, K // G))
    b = r.uniform(-0.1, 0.1, size=(N, K // G))
    c = cat == 1
    s[c] = 0.0
    c = cat == 2
    s[c] = -r.uniform(0.1, 1.0, size=s[c].shape)
    b[c] = -r.uniform(1.0, 4.0, size=b[c].shape)
    c = cat == 5
    s[c] = _signs(r, s[c].shape) * 2.0 ** r.uniform(8, 16, size=s[c].shape)
    b[c] = _signs(r, b[c].shape) * 2.0 ** r.uniform(8, 16, size=b[c].shape)
    s16, b16 = _bf16(s.astype(np.float32)), _bf16(b.astype(np.float32))
    c = cat == 3
    s16[c] = r.integers(1, 0x80, size=s16[c].shape).astype(np.uint16)
    b16[c] = (r.integers(1, 0x80, size=b16[c].shape) | (r.integers(0, 2, size=b16[c].shape) << 15)).astype(np.uint16)
    c = cat == 4
    b16[c] = 0
    qz = q[c]
    qz[:, _slot_mask(K)] = 0
    q[c] = qz
    return dict(q=q, s=s16, b=b16, cat=cat)


def activation(kind: str, K: int, seed: int) -> np.ndarray:
    """One bf16 row [K] (bit patterns) of the given kind."""
    r = _rng(seed, 100 + X_KINDS.index(kind))
    x = r.standard_normal(K).astype(np.float64)
    if kind in ("outlier10", "outlier7"):
        blocks = np.abs(x.reshape(-1, 16))
        blocks[:, OUT_SLOT] = 0.0
        big = blocks.max(axis=1) * (2.0 ** 10 if kind == "outlier10" else 2.0 ** 7)
        x[_slot_mask(K)] = _signs(r, big.shape) * big
    elif kind == "subnormal":
        return (r.integers(1, 0x80, size=K) | (r.integers(0, 2, size=K) << 15)).astype(np.uint16)
    elif kind == "zero_grp":
        x.reshape(-1, 32)[r.integers(0, 2, size=K // 32) == 1] = 0.0
    elif kind == "mixed_sub":
        out = _bf16(x.astype(np.float32))
        k = np.arange(K) % 4 == 3
        out[k] = (r.integers(1, 0x80, size=int(k.sum())) | (r.integers(0, 2, size=int(k.sum())) << 15)).astype(np.uint16)
        return out
    elif kind == "wide20":
        x[_slot_mask(K)] = _signs(r, int(_slot_mask(K).sum())) * 2.0 ** 20
    return _bf16(x.astype(np.float32))


def activations(kinds, K: int, seed: int) -> np.ndarray:
    """bf16 rows [len(kinds)][K], row m of kind kinds[m]."""
    return np.stack([activation(k, K, seed + 7 * m) for m, k in enumerate(kinds)])
