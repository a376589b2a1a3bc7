"""Pins for the CPU oracle: facts fixed by the source pages and by mathematics.

Each ``pin_*`` function takes an oracle implementation (a module exposing the
functions of ``oracle.oracle_np`` / ``oracle.oracle_c``) and raises
AssertionError when the implementation disagrees with the fact.  The same pins
run on both oracle restatements and, in ``test_oracle_mutants.py``, on copies
of the oracle with a planted mistake, to show each pin can fail.

Exact values are computed with ``fractions.Fraction`` from the unpacked inputs
(fp16 patterns decoded by Python's ``struct`` 'e' format, bf16 by ``struct``
'f' on the widened pattern), never from either oracle.
"""
from __future__ import annotations

import json
import os
import struct
from fractions import Fraction

import numpy as np

from int6_quantized_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---- exact helpers -----------------------------------------------------------------

def fr_f16(bits: int) -> Fraction:
    return Fraction(struct.unpack("<e", int(bits).to_bytes(2, "little"))[0])


def fr_bf16(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", (int(bits) << 16).to_bytes(4, "little"))[0])


def f32_of(fr: Fraction) -> np.float32:
    """Nearest-even binary32 of an exact rational that binary64 holds exactly."""
    d = float(fr)
    assert Fraction(d) == fr, "value needs more than 53 bits; pin not applicable"
    return np.float32(d)


def bits32(a) -> np.ndarray:
    return np.asarray(a, np.float32).view(np.uint32)


# ---- bits per weight ([NSS] 'Quant schema update': 4.625 and 6.5625 bpw) -------------

def pin_bpw(impl):
    N, K = 3, 512
    w = synth.int4_weights(11, N, K)
    parts = impl.int4_pack(w["q"], w["sc"], w["zc"], w["ss"], w["zs"])
    assert Fraction(8 * sum(p.nbytes for p in parts), N * K) == Fraction(4625, 1000)
    w = synth.int6_weights(12, N, K)
    parts = impl.int6_pack(w["q"], w["sc"], w["st"])
    assert Fraction(8 * sum(p.nbytes for p in parts), N * K) == Fraction(65625, 10000)
    parts = impl.int6p_pack(w["q"], w["sc"], w["st"])  # the planar layout stores the same bits
    assert Fraction(8 * sum(p.nbytes for p in parts), N * K) == Fraction(65625, 10000)
    for bits in (2, 4, 8):
        w = synth.affine_weights(13, N, K, bits, 64)
        parts = impl.affine_pack(w["q"], w["s"], w["b"], bits, 64)
        # codes plus a 16-bit scale and a 16-bit bias per 64 weights
        assert Fraction(8 * sum(p.nbytes for p in parts), N * K) == bits + Fraction(32, 64)


# ---- hand-derived worked examples ------------------------------------------------------

def pin_golden_layouts(impl):
    g = golden("layout_worked_examples.json")
    K = 256
    # int4 codes / gmeta / steps
    q = np.zeros((1, K), np.uint8)
    q[0, :8] = g["int4_codes"]["q_row"]
    sc = np.zeros((1, K // 32), np.uint8)
    zc = np.zeros((1, K // 32), np.uint8)
    sc[0, 0], zc[0, 0] = g["int4_gmeta"]["sc"], g["int4_gmeta"]["zc"]
    ss = np.array([[g["int4_steps"]["ss_bits"]]], np.uint16)
    zs = np.array([[g["int4_steps"]["zs_bits"]]], np.uint16)
    codes, gmeta, steps = impl.int4_pack(q, sc, zc, ss, zs)
    assert list(codes[0, :4]) == g["int4_codes"]["bytes"]
    assert int(gmeta[0, 0]) == g["int4_gmeta"]["word"]
    assert int(steps[0, 0]) == g["int4_steps"]["word"]
    # int6 codes
    for case in g["int6_codes"]["cases"]:
        q6 = np.zeros((1, K), np.int8)
        q6[0, :4] = case["q"]
        codes, _, _ = impl.int6_pack(q6, np.ones((1, K // 16), np.int8), np.zeros((1, 1), np.uint16))
        assert list(codes[0, :3]) == case["bytes"], case
    # int6 planar codes: every byte not named in a case is zero
    for case in g["int6_planar_codes"]["cases"]:
        q6 = np.zeros((1, 2 * K), np.int8)
        for k, v in case["q_at"].items():
            q6[0, int(k)] = v
        codes, _, _ = impl.int6p_pack(q6, np.ones((1, K // 8), np.int8), np.zeros((1, 2), np.uint16))
        want = np.zeros(3 * 2 * K // 4, np.uint8)
        for i, v in case["bytes_at"].items():
            want[int(i)] = v
        assert np.array_equal(codes[0], want), case
    # affine words
    for case in g["affine_words"]["cases"]:
        b = case["bits"]
        qa = np.zeros((1, K), np.uint8)
        qa[0, :len(case["q"])] = case["q"]
        words, _ = impl.affine_pack(qa, np.zeros((1, K // 64), np.uint16),
                                    np.zeros((1, K // 64), np.uint16), b, 64)
        assert int(words[0, 0]) == case["word"], case


def pin_golden_dequant(impl):
    g = golden("layout_worked_examples.json")
    K = 256
    for case in g["int4_dequant"]["cases"]:
        q = np.full((1, K), case["q"], np.uint8)
        sc = np.full((1, K // 32), case["sc"], np.uint8)
        zc = np.full((1, K // 32), case["zc"], np.uint8)
        ss = np.full((1, 1), case["ss_bits"], np.uint16)
        zs = np.full((1, 1), case["zs_bits"], np.uint16)
        w = impl.int4_dequant(*impl.int4_pack(q, sc, zc, ss, zs))
        assert np.all(w == np.float32(case["w"])), case
    for case in g["int6_dequant"]["cases"]:
        q = np.full((1, K), case["q"], np.int8)
        sc = np.full((1, K // 16), case["sc"], np.int8)
        st = np.full((1, 1), case["st_bits"], np.uint16)
        w = impl.int6_dequant(*impl.int6_pack(q, sc, st))
        assert np.all(w == np.float32(case["w"])), case
    for case in g["affine_dequant"]["cases"]:
        b = case["bits"]
        q = np.full((1, K), case["q"], np.uint8)
        s = np.full((1, K // 64), case["s_bits"], np.uint16)
        bb = np.full((1, K // 64), case["b_bits"], np.uint16)
        w = impl.affine_dequant(*impl.affine_pack(q, s, bb, b, 64), b, 64)
        assert np.all(w == np.float32(case["w"])), case


# ---- exhaustive round trips -------------------------------------------------------------

def pin_roundtrip(impl):
    rng = np.random.default_rng(5)
    # int4: every (even, odd) nibble pair once -> each value at both positions
    a, b = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    q = np.stack([a.ravel(), b.ravel()], -1).reshape(1, 512).astype(np.uint8)
    q = np.concatenate([q, q[:, ::-1]], 0)
    sc = np.arange(256, dtype=np.uint8)[:32].reshape(2, 16)
    zc = (255 - np.arange(32)).astype(np.uint8).reshape(2, 16)
    ss = rng.integers(0, 1 << 16, size=(2, 2), dtype=np.uint16)
    zs = rng.integers(0, 1 << 16, size=(2, 2), dtype=np.uint16)
    out = impl.int4_unpack(*impl.int4_pack(q, sc, zc, ss, zs))
    for x, y in zip((q, sc, zc, ss, zs), out):
        assert np.array_equal(np.asarray(x), np.asarray(y))
    # int6: each of the 64 values at each of the 4 positions of a 3-byte unit
    j, pos = np.arange(256) // 4, np.arange(256) % 4
    q6 = np.stack([((j + 16 * pos + r) % 64) - 32 for r in range(4)]).astype(np.int8)
    q6 = np.concatenate([q6, np.roll(q6, 1, axis=1)], 0)
    sc6 = rng.integers(-128, 128, size=(8, 16), dtype=np.int8)
    st6 = rng.integers(0, 1 << 16, size=(8, 1), dtype=np.uint16)
    out = impl.int6_unpack(*impl.int6_pack(q6, sc6, st6))
    for x, y in zip((q6, sc6, st6), out):
        assert np.array_equal(np.asarray(x), np.asarray(y))
    # int6 planar: the same rows put each value at each position of a nibble pair and a 2-bit quad
    out = impl.int6p_unpack(*impl.int6p_pack(q6, sc6, st6))
    for x, y in zip((q6, sc6, st6), out):
        assert np.array_equal(np.asarray(x), np.asarray(y))
    # affine: each value at each of the P positions of a word
    for bits in (2, 4, 8):
        P, V = 32 // bits, 1 << bits
        K = 256 * max(1, V * P // 256)
        qa = np.stack([(np.arange(K) // P + r) % V for r in range(P)]).astype(np.uint8)
        s = rng.integers(0, 1 << 16, size=(P, K // 64), dtype=np.uint16)
        bb = rng.integers(0, 1 << 16, size=(P, K // 64), dtype=np.uint16)
        out = impl.affine_unpack(*impl.affine_pack(qa, s, bb, bits, 64), bits, 64)
        for x, y in zip((qa, s, bb), out):
            assert np.array_equal(np.asarray(x), np.asarray(y)), bits


# ---- exact rational dequantisation -------------------------------------------------------

def pin_int4_exact(impl, N=3, K=512, seed=21):
    """With config-range steps, q - zero is exact, so w is the binary32 rounding of the
    exact (q - zc*zs) * (sc*ss)."""
    w = synth.int4_weights(seed, N, K)
    # include extreme codes in every position class
    w["q"][0, :4] = [0, 15, 0, 15]
    w["sc"][0, :2] = [0, 255]
    w["zc"][0, :2] = [255, 0]
    got = impl.int4_dequant(*impl.int4_pack(w["q"], w["sc"], w["zc"], w["ss"], w["zs"]))
    rng = np.random.default_rng(seed)
    idx = [(0, k) for k in range(64)] + [(int(rng.integers(N)), int(rng.integers(K))) for _ in range(300)]
    for n, k in idx:
        g, j = k // 32, k // 256
        S = int(w["sc"][n, g]) * fr_f16(w["ss"][n, j])
        Z = int(w["zc"][n, g]) * fr_f16(w["zs"][n, j])
        exact = (int(w["q"][n, k]) - Z) * S
        # value equality: bit-exact for nonzero values, and +0 == -0 when the scale is 0
        assert got[n, k] == f32_of(exact), (n, k)


def pin_int6_exact(impl, N=3, K=512, seed=22):
    """int6 needs no rounding at all: w equals the exact q * sc * st (dense and planar storage)."""
    w = synth.int6_weights(seed, N, K)
    w["q"][0, :4] = [-32, 31, 0, -1]
    w["sc"][0, :2] = [-128, 127]
    rng = np.random.default_rng(seed)
    idx = [(0, k) for k in range(64)] + [(int(rng.integers(N)), int(rng.integers(K))) for _ in range(300)]
    for pack, dequant in ((impl.int6_pack, impl.int6_dequant), (impl.int6p_pack, impl.int6p_dequant)):
        got = dequant(*pack(w["q"], w["sc"], w["st"]))
        for n, k in idx:
            exact = int(w["q"][n, k]) * int(w["sc"][n, k // 16]) * fr_f16(w["st"][n, k // 256])
            assert Fraction(float(got[n, k])) == exact, (n, k)


def pin_affine_exact(impl, N=3, K=512, seed=23):
    """q*scale is exact, so w is the binary32 rounding of the exact q*s + b."""
    for bits in (2, 4, 8):
        w = synth.affine_weights(seed, N, K, bits, 64)
        got = impl.affine_dequant(*impl.affine_pack(w["q"], w["s"], w["b"], bits, 64), bits, 64)
        rng = np.random.default_rng(seed + bits)
        idx = [(0, k) for k in range(64)] + [(int(rng.integers(N)), int(rng.integers(K))) for _ in range(200)]
        for n, k in idx:
            exact = int(w["q"][n, k]) * fr_bf16(w["s"][n, k // 64]) + fr_bf16(w["b"][n, k // 64])
            assert bits32(got[n, k]) == bits32(f32_of(exact)), (bits, n, k)


# ---- special cases ----------------------------------------------------------------------

def pin_special_cases(impl):
    K = 256
    rng = np.random.default_rng(31)
    # int6 is odd-symmetric and has no zero point: w(-q) = -w(q), w(0) = 0
    q = rng.integers(-31, 32, size=(2, K)).astype(np.int8)
    sc = rng.integers(-127, 128, size=(2, K // 16)).astype(np.int8)
    st = np.array([[0x2A00], [0x1C00]], np.uint16)
    w_pos = impl.int6_dequant(*impl.int6_pack(q, sc, st))
    w_neg = impl.int6_dequant(*impl.int6_pack(-q, sc, st))
    assert np.array_equal(w_neg, -w_pos)
    assert np.all((w_pos == 0) == ((q == 0) | (np.repeat(sc, 16, 1) == 0)))
    # the planar storage holds the same codes: its weights equal the dense layout's, and its
    # low plane is byte for byte the int4 nibble packing of the codes' low 4 bits
    assert np.array_equal(impl.int6p_dequant(*impl.int6p_pack(q, sc, st)), w_pos)
    lo4 = (q.view(np.uint8) & 0xF).astype(np.uint8)
    nib = impl.int4_pack(lo4, np.zeros((2, 8), np.uint8), np.zeros((2, 8), np.uint8),
                         np.zeros((2, 1), np.uint16), np.zeros((2, 1), np.uint16))[0]
    assert np.array_equal(impl.int6p_pack(q, sc, st)[0][:, :128], nib)
    # int4 with zero code 0 reduces to q * scale
    q4 = rng.integers(0, 16, size=(2, K)).astype(np.uint8)
    sc4 = rng.integers(0, 256, size=(2, 8)).astype(np.uint8)
    zc4 = np.zeros((2, 8), np.uint8)
    ss = np.array([[0x1C00], [0x2A55]], np.uint16)
    zs = np.array([[0x2400], [0x2600]], np.uint16)
    w4 = impl.int4_dequant(*impl.int4_pack(q4, sc4, zc4, ss, zs))
    for n in range(2):
        S = np.repeat(sc4[n].astype(np.float64), 32) * float(fr_f16(ss[n, 0]))
        assert np.array_equal(w4[n], (q4[n] * S).astype(np.float32))
    # power-of-two steps with unit codes: w = (q - zs) * ss exactly
    ones = np.ones((2, 8), np.uint8)
    w4 = impl.int4_dequant(*impl.int4_pack(q4, ones, ones, np.full((2, 1), 0x2000, np.uint16),
                                           np.full((2, 1), 0x3800, np.uint16)))
    assert np.array_equal(w4, ((q4.astype(np.float64) - 0.5) * 2.0 ** -7).astype(np.float32))
    # affine with scale 1 and bias 0 returns the codes
    for bits in (2, 4, 8):
        qa = rng.integers(0, 1 << bits, size=(2, K)).astype(np.uint8)
        one = np.full((2, K // 64), 0x3F80, np.uint16)
        zero = np.zeros((2, K // 64), np.uint16)
        wa = impl.affine_dequant(*impl.affine_pack(qa, one, zero, bits, 64), bits, 64)
        assert np.array_equal(wa, qa.astype(np.float32))


# ---- the layer (binary64 matmul) ----------------------------------------------------------

def pin_matmul(impl):
    rng = np.random.default_rng(41)
    # brute-force rational dot products on tiny shapes
    for M, N, K in ((1, 1, 256), (3, 8, 256), (2, 5, 512)):
        x = synth.activations(int(rng.integers(1 << 30)), M, K)
        w = rng.standard_normal(size=(N, K)).astype(np.float32)
        y = impl.matmul_f64(x, w)
        assert y.shape == (M, N)
        for m in range(M):
            xf = [fr_bf16(v) for v in x[m]]
            for n in range(N):
                terms = [a * Fraction(float(b)) for a, b in zip(xf, w[n])]
                exact = sum(terms)
                bound = Fraction(K + 1, 2 ** 53) * sum(abs(t) for t in terms)
                assert abs(Fraction(float(y[m, n])) - exact) <= bound, (M, N, K, m, n)
    # power-of-two scaling of x is exact end to end; row permutations permute columns
    M, N, K = 2, 6, 256
    x = synth.activations(7, M, K)
    w = rng.standard_normal(size=(N, K)).astype(np.float32)
    x2 = (x.astype(np.uint32) + np.where((x & 0x7F80) != 0, 0x80, 0)).astype(np.uint16)  # *2 in bf16
    y, y2 = impl.matmul_f64(x, w), impl.matmul_f64(x2, w)
    assert np.array_equal(y2, 2 * y)
    perm = rng.permutation(N)
    assert np.array_equal(impl.matmul_f64(x, w[perm]), y[:, perm])
    # linearity in x with disjoint supports: y(x_a + x_b) = y(x_a) + y(x_b) within rounding
    xa = x.copy(); xa[:, K // 2:] = 0
    xb = x.copy(); xb[:, :K // 2] = 0
    assert np.allclose(impl.matmul_f64(xa, w) + impl.matmul_f64(xb, w), y, rtol=1e-12, atol=1e-12)


# ---- metadata encoder ([NSS] 'Quant schema update'; [REV] 'Correctness' 1, 'Things done well') --

def fr_round_f32(fr: Fraction) -> Fraction:
    """Nearest-even binary32 of an exact positive rational in the normal range, computed exactly."""
    assert fr > 0
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    assert -126 <= e <= 127, "outside the binary32 normal range"
    ulp = Fraction(2) ** (e - 23)
    m = fr / ulp  # in [2^23, 2^24)
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return lo * ulp


def fr_round_f16_bits(fr: Fraction) -> int:
    """Binary16 bit pattern nearest (ties to even) to a value that binary64 holds exactly."""
    d = float(fr)
    assert Fraction(d) == fr
    return struct.unpack("<H", struct.pack("<e", d))[0]


def _encode_expected(v: np.ndarray, per: int, top: int, signed: bool):
    """Codes and step bits of one field, derived with exact rationals from the encoder's definition."""
    N, G = v.shape
    codes = np.zeros((N, G), np.int64)
    steps = np.zeros((N, G // per), np.int64)
    for r in range(N):
        for b in range(G // per):
            block = [Fraction(float(x)) for x in v[r, b * per:(b + 1) * per]]
            m = max(abs(x) for x in block) if signed else max(block)
            step_bits = fr_round_f16_bits(fr_round_f32(m / top)) if m > 0 else 0
            steps[r, b] = step_bits
            sf = fr_f16(step_bits)
            for i, x in enumerate(block):
                if sf == 0 or x == 0:
                    c = 0
                else:
                    qv = fr_round_f32(abs(x) / sf) * (1 if x > 0 else -1)
                    c = round(qv)  # Fraction rounds half to even
                codes[r, b * per + i] = max(-top, min(top, c)) if signed else max(0, min(255, c))
    return codes, steps


def pin_encoder_golden(impl):
    g = golden("meta_encoder_worked_example.json")
    codes, steps = impl.encode_u8_per_super(np.array([g["values"]], np.float32), 8)
    assert codes.ravel().tolist() == g["codes"], codes
    assert int(steps[0, 0]) == g["step_bits"], hex(int(steps[0, 0]))


def pin_encoder_exact(impl, seed=31):
    rng = np.random.default_rng(seed)
    # int4 fields: scales ~ 1e-4..1e-2 and zero points 0..15 (code units), 4 super-blocks per row,
    # one all-zero super-block
    sc = rng.uniform(1e-4, 1e-2, (3, 32)).astype(np.float32)
    zp = (rng.uniform(0, 15, (3, 32)) * (rng.random((3, 32)) > 0.1)).astype(np.float32)
    zp[1, 8:16] = 0.0
    for v in (sc, zp):
        c, s = impl.encode_u8_per_super(v, 8)
        ce, se = _encode_expected(v, 8, 255, False)
        assert np.array_equal(np.asarray(c, np.int64), ce)
        assert np.array_equal(np.asarray(s, np.int64), se)
    # int6 field: signed scales, 16 groups per super-block
    s6 = (rng.uniform(1e-4, 1e-2, (2, 32)) * rng.choice([-1, 1], (2, 32))).astype(np.float32)
    c, s = impl.encode_i8_per_super(s6, 16)
    ce, se = _encode_expected(s6, 16, 127, True)
    assert np.array_equal(np.asarray(c, np.int64), ce)
    assert np.array_equal(np.asarray(s, np.int64), se)


def pin_encoder_agreement(impl, seed=32):
    """Encode/decode agreement: every value lies within half a step (plus the binary32 rounding of
    the quotient) of code * step_f, the block max encodes to 254 or 255, and int6 codes are odd in v."""
    rng = np.random.default_rng(seed)
    v = rng.uniform(0, 3, (4, 64)).astype(np.float32)
    c, s = impl.encode_u8_per_super(v, 8)
    sf = np.repeat(np.asarray(s, np.uint16).view(np.float16).astype(np.float64), 8, 1)
    err = np.abs(v.astype(np.float64) - np.asarray(c, np.float64) * sf)
    assert np.all(err <= sf * (0.5 + 2.0 ** -15)), err.max()
    vb = v.reshape(4, 8, 8)
    cb = np.asarray(c).reshape(4, 8, 8)
    assert np.all(cb[np.arange(4)[:, None], np.arange(8)[None, :], vb.argmax(2)] >= 254)
    c6, _ = impl.encode_i8_per_super(v - 1.5, 16)
    c6n, _ = impl.encode_i8_per_super(-(v - 1.5), 16)
    assert np.array_equal(np.asarray(c6, np.int64), -np.asarray(c6n, np.int64))


def pin_snr(impl):
    w = np.ones(1000)
    assert abs(impl.snr_db(w, 0.9 * w) - 20.0) < 1e-9  # 10 log10(1 / 0.01)
    assert abs(impl.snr_db(w, w + 1e-3) - 60.0) < 1e-6
