"""Second, independent restatement of the oracle in NumPy.

Test infrastructure only (the product path never imports it).  It computes the
same things as ``oracle.c`` by other means -- NumPy's own binary16 type for the
fp16 steps, vectorised bit operations for the packing, float32 ufuncs for the
dequantisation and a float64 matrix product for the layer -- so that the two
restatements can pin each other.

Sources, cited by page title and section:
  [NSS] ExecuTorch PR "[cuda] Nestest Superscale Quantization for CUDA Weights
        (int4 / int6)", section "Quant schema update".
  [MTL] Hugging Face Transformers docs, "Metal" quantization page.
  [REV] the same ExecuTorch PR, the review ("PR Review: Superscale
        Quantization for CUDA Weights"), "Correctness" note 1 and "Things
        done well" (encode/decode agreement); "Ablation study" (SNR).
"""
from __future__ import annotations

import numpy as np

f32 = np.float32


def f32_from_f16_bits(h) -> np.ndarray:
    return np.ascontiguousarray(h, np.uint16).view(np.float16).astype(np.float32)


def f32_from_bf16_bits(b) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_from_f32(a) -> np.ndarray:
    """Nearest-even rounding of binary32 values to bfloat16 bit patterns."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, np.float32))
    return np.where(nan, np.uint16(0x7FC0), r)


# ---- int4 nested superscale ([NSS]: group 32, super-block 256) ------------------

def int4_pack(q, sc, zc, ss, zs):
    q = np.asarray(q, np.uint8) & 0xF
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    gmeta = (np.asarray(sc, np.uint16) | (np.asarray(zc, np.uint16) << 8)).astype(np.uint16)
    steps = (np.asarray(ss, np.uint32) | (np.asarray(zs, np.uint32) << 16)).astype(np.uint32)
    return codes, gmeta, steps


def int4_unpack(codes, gmeta, steps):
    codes = np.asarray(codes, np.uint8)
    N = codes.shape[0]
    q = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(N, -1)
    gmeta = np.asarray(gmeta, np.uint16)
    steps = np.asarray(steps, np.uint32)
    return (q, (gmeta & 0xFF).astype(np.uint8), (gmeta >> 8).astype(np.uint8),
            (steps & 0xFFFF).astype(np.uint16), (steps >> 16).astype(np.uint16))


def int4_dequant(codes, gmeta, steps):
    q, sc, zc, ss, zs = int4_unpack(codes, gmeta, steps)
    scale_step = np.repeat(f32_from_f16_bits(ss), 8, axis=1)   # per group of 32
    zero_step = np.repeat(f32_from_f16_bits(zs), 8, axis=1)
    S = sc.astype(f32) * scale_step          # scale = code x step
    Z = zc.astype(f32) * zero_step           # zero  = code x step
    t = q.astype(f32) - np.repeat(Z, 32, axis=1)
    return (t * np.repeat(S, 32, axis=1)).astype(f32)


# ---- int6 symmetric ([NSS]: group 16, super-block 256) ---------------------------

def int6_pack(q, sc, st):
    q = np.asarray(q, np.int8)
    N, K = q.shape
    f = (q.view(np.uint8) & 0x3F).astype(np.uint32).reshape(N, K // 4, 4)
    u = f[..., 0] | (f[..., 1] << 6) | (f[..., 2] << 12) | (f[..., 3] << 18)
    b = np.stack([u & 0xFF, (u >> 8) & 0xFF, (u >> 16) & 0xFF], axis=-1)
    return (b.reshape(N, 3 * K // 4).astype(np.uint8), np.asarray(sc, np.int8).copy(),
            np.asarray(st, np.uint16).copy())


def int6_unpack(codes, gmeta, steps):
    codes = np.asarray(codes, np.uint8)
    N = codes.shape[0]
    b = codes.reshape(N, -1, 3).astype(np.uint32)
    u = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    f = np.stack([(u >> (6 * i)) & 0x3F for i in range(4)], axis=-1).reshape(N, -1)
    q = (f.astype(np.int16) - 64 * (f >= 32)).astype(np.int8)
    return q, np.asarray(gmeta, np.int8).copy(), np.asarray(steps, np.uint16).copy()


def int6_dequant(codes, gmeta, steps):
    q, sc, st = int6_unpack(codes, gmeta, steps)
    step = np.repeat(f32_from_f16_bits(st), 16, axis=1)       # per group of 16
    S = sc.astype(f32) * step                                  # scale = code x step
    return (q.astype(f32) * np.repeat(S, 16, axis=1)).astype(f32)


# ---- int6 planar ([REV] "Correctness" note 2: a 4-bit plane and a 2-bit plane) -------
# Per 256-weight super-block of a row: 128 bytes of low nibbles (even weight in the low nibble),
# then 64 bytes of the codes' bits 4-5 (weight i at bits 2*(i%4) of byte 128 + i/4).

def int6p_pack(q, sc, st):
    q = np.asarray(q, np.int8)
    N, K = q.shape
    f = (q.view(np.uint8) & 0x3F).reshape(N, K // 256, 256)
    lo, hi = f & 0xF, f >> 4
    lo_plane = lo[..., 0::2] | (lo[..., 1::2] << 4)
    hi_plane = hi[..., 0::4] | (hi[..., 1::4] << 2) | (hi[..., 2::4] << 4) | (hi[..., 3::4] << 6)
    codes = np.concatenate([lo_plane, hi_plane], axis=-1).reshape(N, 3 * K // 4).astype(np.uint8)
    return codes, np.asarray(sc, np.int8).copy(), np.asarray(st, np.uint16).copy()


def int6p_unpack(codes, gmeta, steps):
    codes = np.asarray(codes, np.uint8)
    N = codes.shape[0]
    blk = codes.reshape(N, -1, 192)
    lo = np.stack([blk[..., :128] & 0xF, blk[..., :128] >> 4], axis=-1).reshape(N, -1, 256)
    hi = np.stack([(blk[..., 128:] >> (2 * i)) & 0x3 for i in range(4)], axis=-1).reshape(N, -1, 256)
    f = (lo | (hi << 4)).reshape(N, -1)
    q = (f.astype(np.int16) - 64 * (f >= 32)).astype(np.int8)
    return q, np.asarray(gmeta, np.int8).copy(), np.asarray(steps, np.uint16).copy()


def int6p_dequant(codes, gmeta, steps):
    q, sc, st = int6p_unpack(codes, gmeta, steps)
    step = np.repeat(f32_from_f16_bits(st), 16, axis=1)       # per group of 16
    S = sc.astype(f32) * step                                  # scale = code x step
    return (q.astype(f32) * np.repeat(S, 16, axis=1)).astype(f32)


# ---- uint32 affine ([MTL]) -------------------------------------------------------

def affine_pack(q, s, b, bits: int, G: int):
    q = np.asarray(q, np.uint8)
    N, K = q.shape
    P = 32 // bits
    mask = (1 << bits) - 1
    f = (q & mask).astype(np.uint32).reshape(N, K // P, P)
    shifts = (bits * np.arange(P, dtype=np.uint32))
    words = np.bitwise_or.reduce(f << shifts, axis=-1).astype(np.uint32)
    gmeta = (np.asarray(s, np.uint32) | (np.asarray(b, np.uint32) << 16)).astype(np.uint32)
    return words, gmeta


def affine_unpack(codes, gmeta, bits: int, G: int):
    codes = np.asarray(codes, np.uint32)
    N = codes.shape[0]
    P = 32 // bits
    shifts = (bits * np.arange(P, dtype=np.uint32))
    q = ((codes[..., None] >> shifts) & ((1 << bits) - 1)).reshape(N, -1).astype(np.uint8)
    gmeta = np.asarray(gmeta, np.uint32)
    return q, (gmeta & 0xFFFF).astype(np.uint16), (gmeta >> 16).astype(np.uint16)


def affine_dequant(codes, gmeta, bits: int, G: int):
    q, s, b = affine_unpack(codes, gmeta, bits, G)
    scale = np.repeat(f32_from_bf16_bits(s), G, axis=1)
    bias = np.repeat(f32_from_bf16_bits(b), G, axis=1)
    p = q.astype(f32) * scale                 # q * scale
    return (p + bias).astype(f32)             # + bias


# ---- the linear layer -------------------------------------------------------------

def matmul_f64(x_bf16, w):
    """y = x . w^T with x given as bf16 bit patterns, in binary64."""
    x = f32_from_bf16_bits(x_bf16).astype(np.float64)
    return x @ np.asarray(w, np.float32).astype(np.float64).T


# ---- metadata encoder ([NSS] "Quant schema update"; [REV] "Correctness" 1) ----------
# Per 256-weight super-block, each per-group float field becomes a code times one fp16 step.

def encode_u8_per_super(v, groups_per_super: int):
    """int4 scale or zero field -> (u8 codes [N][G], fp16 step bits [N][G/groups_per_super]).

    Steps, as the review describes the encoder: block_max = the super-block's max (a max, not an
    absmax; the field must be non-negative, checked here), step = fp16(block_max / 255) with the
    division in float32, code = clamp(round_half_even(v / step_f), 0, 255) where step_f is the
    fp16-rounded step (so encoder and decoder reconstruct with the same step).  A super-block
    whose max is 0 gets step 0 and codes 0 (the pages do not say; the plainest reading)."""
    v = np.asarray(v, np.float32)
    if not np.isfinite(v).all() or (v < 0).any():
        raise ValueError("int4 metadata fields must be finite and non-negative")
    N, G = v.shape
    vb = v.reshape(N, G // groups_per_super, groups_per_super)
    block_max = vb.max(axis=2)
    step16 = (block_max / f32(255)).astype(np.float16)
    step_f = step16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(vb / step_f)
    q = np.where(step_f > 0, q, 0)
    codes = np.clip(q, 0, 255).astype(np.uint8)
    return codes.reshape(N, G), step16.view(np.uint16)


def encode_i8_per_super(v, groups_per_super: int):
    """int6 scale field -> (i8 codes [N][G], fp16 step bits [N][G/groups_per_super]).

    The pages give no int6 encoder; the symmetric counterpart of the int4 one is taken:
    step = fp16(max|v| / 127), code = clamp(round_half_even(v / step_f), -127, 127)."""
    v = np.asarray(v, np.float32)
    if not np.isfinite(v).all():
        raise ValueError("int6 scale field must be finite")
    N, G = v.shape
    vb = v.reshape(N, G // groups_per_super, groups_per_super)
    block_max = np.abs(vb).max(axis=2)
    step16 = (block_max / f32(127)).astype(np.float16)
    step_f = step16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(vb / step_f)
    q = np.where(step_f > 0, q, 0)
    codes = np.clip(q, -127, 127).astype(np.int8)
    return codes.reshape(N, G), step16.view(np.uint16)


def snr_db(w, w_hat) -> float:
    """Whole-tensor signal-to-noise ratio in dB, 10 log10(sum w^2 / sum (w - w_hat)^2), as the
    ablation study reports it (formula not printed there; the standard definition)."""
    w = np.asarray(w, np.float64)
    e = w - np.asarray(w_hat, np.float64)
    return float(10.0 * np.log10((w * w).sum() / (e * e).sum()))
