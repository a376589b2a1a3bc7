"""Each pin can fail: plant one plausible mistake in a copy of the NumPy oracle
and check that at least one pin rejects it (CPU only; nothing here runs on a GPU)."""
import types

import numpy as np
import pytest

from oracle import oracle_np as O
from tests import oracle_pins as P

ALL_PINS = [P.pin_bpw, P.pin_golden_layouts, P.pin_golden_dequant, P.pin_roundtrip,
            P.pin_int4_exact, P.pin_int6_exact, P.pin_affine_exact, P.pin_special_cases,
            P.pin_matmul]
f32 = np.float32


def mutant(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(O, k) for k in dir(O) if not k.startswith("_")})
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


def _int4_parts(codes, gmeta, steps):
    q, sc, zc, ss, zs = O.int4_unpack(codes, gmeta, steps)
    return (q, sc, zc, np.repeat(O.f32_from_f16_bits(ss), 8, 1), np.repeat(O.f32_from_f16_bits(zs), 8, 1))


def int4_swapped_steps(codes, gmeta, steps):
    q, sc, zc, ss, zs = _int4_parts(codes, gmeta, steps)
    S, Z = sc.astype(f32) * zs, zc.astype(f32) * ss
    return ((q.astype(f32) - np.repeat(Z, 32, 1)) * np.repeat(S, 32, 1)).astype(f32)


def int4_scale_then_shift(codes, gmeta, steps):
    q, sc, zc, ss, zs = _int4_parts(codes, gmeta, steps)
    S, Z = sc.astype(f32) * ss, zc.astype(f32) * zs
    return (q.astype(f32) * np.repeat(S, 32, 1) - np.repeat(Z, 32, 1)).astype(f32)


def int4_group16(codes, gmeta, steps):
    q, sc, zc, ss, zs = _int4_parts(codes, gmeta, steps)
    S, Z = sc.astype(f32) * ss, zc.astype(f32) * zs
    K = q.shape[1]
    S16 = np.repeat(S, 16, 1)[:, :K] if S.shape[1] * 16 >= K else np.repeat(np.repeat(S, 16, 1), 2, 1)
    Z16 = np.repeat(Z, 16, 1)
    S16 = np.concatenate([S16, S16], 1)[:, :K]
    Z16 = np.concatenate([Z16, Z16], 1)[:, :K]
    return ((q.astype(f32) - Z16) * S16).astype(f32)


def int4_pack_high_first(q, sc, zc, ss, zs):
    codes, gmeta, steps = O.int4_pack(q, sc, zc, ss, zs)
    return ((codes >> 4) | (codes << 4)).astype(np.uint8), gmeta, steps


def int4_pack_wide_meta(q, sc, zc, ss, zs):
    codes, gmeta, steps = O.int4_pack(q, sc, zc, ss, zs)
    return codes, np.concatenate([gmeta, gmeta], 1), steps


def int6_unpack_no_sign(codes, gmeta, steps):
    q, sc, st = O.int6_unpack(codes, gmeta, steps)
    return (q.view(np.uint8) & 0x3F).astype(np.int8), sc, st


def int6_dequant_no_sign(codes, gmeta, steps):
    q, sc, st = int6_unpack_no_sign(codes, gmeta, steps)
    S = sc.astype(f32) * np.repeat(O.f32_from_f16_bits(st), 16, 1)
    return (q.astype(f32) * np.repeat(S, 16, 1)).astype(f32)


def int6_dequant_group32(codes, gmeta, steps):
    q, sc, st = O.int6_unpack(codes, gmeta, steps)
    S = sc.astype(f32) * np.repeat(O.f32_from_f16_bits(st), 16, 1)
    K = q.shape[1]
    return (q.astype(f32) * np.repeat(S, 32, 1)[:, :K]).astype(f32)


def int6p_pack_planes_swapped(q, sc, st):
    codes, gmeta, steps = O.int6p_pack(q, sc, st)
    N = codes.shape[0]
    blk = codes.reshape(N, -1, 192)
    return np.concatenate([blk[..., 128:], blk[..., :128]], -1).reshape(N, -1), gmeta, steps


def int6p_unpack_planes_swapped(codes, gmeta, steps):
    N = codes.shape[0]
    blk = np.asarray(codes, np.uint8).reshape(N, -1, 192)
    return O.int6p_unpack(np.concatenate([blk[..., 64:], blk[..., :64]], -1).reshape(N, -1), gmeta, steps)


def int6p_dequant_planes_swapped(codes, gmeta, steps):
    q, sc, st = int6p_unpack_planes_swapped(codes, gmeta, steps)
    return O.int6_dequant(*O.int6_pack(q, sc, st))


def int6p_pack_high_nibble_first(q, sc, st):
    codes, gmeta, steps = O.int6p_pack(q, sc, st)
    N = codes.shape[0]
    blk = codes.reshape(N, -1, 192).copy()
    blk[..., :128] = (blk[..., :128] >> 4) | (blk[..., :128] << 4)
    return blk.reshape(N, -1), gmeta, steps


def affine_bias_first(codes, gmeta, bits, G):
    q, s, b = O.affine_unpack(codes, gmeta, bits, G)
    sc, bi = np.repeat(O.f32_from_bf16_bits(s), G, 1), np.repeat(O.f32_from_bf16_bits(b), G, 1)
    return ((q.astype(f32) + bi) * sc).astype(f32)


def affine_pack_msb_first(q, s, b, bits, G):
    words, gmeta = O.affine_pack(q, s, b, bits, G)
    P = 32 // bits
    out = np.zeros_like(words)
    for i in range(P):
        out |= ((words >> (bits * i)) & ((1 << bits) - 1)) << (bits * (P - 1 - i))
    return out, gmeta


def matmul_drops_last_k(x_bf16, w):
    return O.matmul_f64(np.asarray(x_bf16)[:, :-1], np.asarray(w)[:, :-1])


def matmul_f32_accumulate(x_bf16, w):
    x = O.f32_from_bf16_bits(x_bf16)
    return (x @ np.asarray(w, np.float32).T).astype(np.float64)


MUTANTS = {
    "int4 steps swapped": mutant(int4_dequant=int4_swapped_steps),
    "int4 q*scale - zero": mutant(int4_dequant=int4_scale_then_shift),
    "int4 group of 16": mutant(int4_dequant=int4_group16),
    "int4 high nibble first": mutant(int4_pack=int4_pack_high_first),
    "int4 metadata too wide": mutant(int4_pack=int4_pack_wide_meta),
    "int6 no sign extension": mutant(int6_unpack=int6_unpack_no_sign, int6_dequant=int6_dequant_no_sign),
    "int6 group of 32": mutant(int6_dequant=int6_dequant_group32),
    "int6 planar: 2-bit plane first": mutant(int6p_pack=int6p_pack_planes_swapped,
                                             int6p_unpack=int6p_unpack_planes_swapped,
                                             int6p_dequant=int6p_dequant_planes_swapped),
    "int6 planar: high nibble first": mutant(int6p_pack=int6p_pack_high_nibble_first),
    "affine (q+b)*s": mutant(affine_dequant=affine_bias_first),
    "affine msb first": mutant(affine_pack=affine_pack_msb_first),
    "matmul drops a term": mutant(matmul_f64=matmul_drops_last_k),
    "matmul fp32 accumulate": mutant(matmul_f64=matmul_f32_accumulate),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    impl = MUTANTS[name]
    failed = []
    for pin in ALL_PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {name}"
