"""The oracle, pinned to facts fixed outside itself (CPU only).

Both restatements (C99 via ctypes, and NumPy) must satisfy every pin, and must
agree with each other bit for bit on packing and dequantisation.
"""
import struct

import numpy as np
import pytest

from int6_quantized_linear_b200 import synth
from oracle import oracle_c, oracle_np
from tests import oracle_pins as P

IMPLS = [pytest.param(oracle_c, id="c"), pytest.param(oracle_np, id="numpy")]


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("pin", [P.pin_bpw, P.pin_golden_layouts, P.pin_golden_dequant,
                                 P.pin_roundtrip, P.pin_int4_exact, P.pin_int6_exact,
                                 P.pin_affine_exact, P.pin_special_cases, P.pin_matmul],
                         ids=lambda f: f.__name__)
def test_pin(impl, pin):
    pin(impl)


# ---- scalar conversions -----------------------------------------------------------------

def test_f16_conversion_exhaustive():
    """Every binary16 pattern decodes to the value Python's struct 'e' decoder gives."""
    for h in range(1 << 16):
        ref = struct.unpack("<e", h.to_bytes(2, "little"))[0]
        got = oracle_c.f32_from_f16(h)
        if ref != ref:
            assert got != got
        else:
            assert got == ref and (np.signbit(got) == np.signbit(ref)), h
    allbits = np.arange(1 << 16, dtype=np.uint16)
    a = oracle_np.f32_from_f16_bits(allbits)
    b = np.array([oracle_c.f32_from_f16(int(h)) for h in allbits[::97]], np.float32)
    assert np.array_equal(a[::97].view(np.uint32)[~np.isnan(a[::97])],
                          b.view(np.uint32)[~np.isnan(b)])


def _bf16_nearest_even(x: float) -> int:
    """Independent reference: nearest-even over the bfloat16 grid by exact comparison."""
    from fractions import Fraction
    f = Fraction(x)
    u = np.float32(x).view(np.uint32)
    lo_bits = int(u) >> 16
    lo = Fraction(float(np.array([lo_bits << 16], np.uint32).view(np.float32)[0]))
    hi_bits = lo_bits + 1
    hi = Fraction(float(np.array([hi_bits << 16], np.uint32).view(np.float32)[0]))
    dlo, dhi = abs(f - lo), abs(hi - f)
    if dlo < dhi:
        return lo_bits
    if dhi < dlo:
        return hi_bits
    return lo_bits if lo_bits % 2 == 0 else hi_bits


def test_bf16_rounding():
    rng = np.random.default_rng(3)
    vals = list(rng.standard_normal(2000).astype(np.float32))
    vals += list((rng.standard_normal(500) * 1e30).astype(np.float32))
    vals += list((rng.standard_normal(500) * 1e-30).astype(np.float32))
    # exact ties: low 16 bits = 0x8000 with odd and even kept parts
    for base in (0x3F80, 0x3F81, 0xBF82, 0x4123, 0x0001):
        vals.append(np.array([(base << 16) | 0x8000], np.uint32).view(np.float32)[0])
    for v in vals:
        want = _bf16_nearest_even(float(v))
        assert oracle_c.bf16_from_f32(v) == want, v
        assert int(oracle_np.bf16_bits_from_f32(np.array([v], np.float32))[0]) == want, v
    # rounding straight from binary64 agrees with the two-step path when binary32 is exact
    y = rng.standard_normal(100).astype(np.float32).astype(np.float64)
    assert np.array_equal(oracle_c.bf16_from_f64(y), oracle_np.bf16_bits_from_f32(y.astype(np.float32)))
    assert oracle_c.bf16_from_f64(np.array([3.0e38 * 1.2]))[0] == 0x7F80     # overflows to inf
    assert oracle_c.bf16_from_f64(np.array([-0.0]))[0] == 0x8000


# ---- the two restatements agree ------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 256), (7, 512), (33, 1024)])
def test_c_numpy_agree_int4(N, K):
    w = synth.int4_weights(N * 7 + K, N, K)
    pc = oracle_c.int4_pack(w["q"], w["sc"], w["zc"], w["ss"], w["zs"])
    pn = oracle_np.int4_pack(w["q"], w["sc"], w["zc"], w["ss"], w["zs"])
    for a, b in zip(pc, pn):
        assert np.array_equal(a, b)
    assert np.array_equal(oracle_c.int4_dequant(*pc).view(np.uint32),
                          oracle_np.int4_dequant(*pn).view(np.uint32))


@pytest.mark.parametrize("N,K", [(1, 256), (7, 512), (33, 1024)])
def test_c_numpy_agree_int6(N, K):
    w = synth.int6_weights(N * 5 + K, N, K)
    pc = oracle_c.int6_pack(w["q"], w["sc"], w["st"])
    pn = oracle_np.int6_pack(w["q"], w["sc"], w["st"])
    for a, b in zip(pc, pn):
        assert np.array_equal(a, b)
    assert np.array_equal(oracle_c.int6_dequant(*pc).view(np.uint32),
                          oracle_np.int6_dequant(*pn).view(np.uint32))


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_c_numpy_agree_affine(bits, G):
    N, K = 9, 512
    w = synth.affine_weights(bits * 100 + G, N, K, bits, G)
    pc = oracle_c.affine_pack(w["q"], w["s"], w["b"], bits, G)
    pn = oracle_np.affine_pack(w["q"], w["s"], w["b"], bits, G)
    for a, b in zip(pc, pn):
        assert np.array_equal(a, b)
    assert np.array_equal(oracle_c.affine_dequant(*pc, bits, G).view(np.uint32),
                          oracle_np.affine_dequant(*pn, bits, G).view(np.uint32))


def test_c_numpy_agree_matmul():
    x = synth.activations(9, 3, 1024)
    w = np.random.default_rng(9).standard_normal((40, 1024)).astype(np.float32)
    yc, yn = oracle_c.matmul_f64(x, w), oracle_np.matmul_f64(x, w)
    assert np.allclose(yc, yn, rtol=1e-12, atol=1e-12)


def test_synth_prefix_property():
    """Activations for a smaller batch are the first rows of a larger draw."""
    a8 = synth.activations(1, 8, 512)
    for m in (1, 4):
        assert np.array_equal(synth.activations(1, m, 512), a8[:m])
    w = synth.int6_weights(2, 4, 256)
    assert not np.any(w["sc"] == 0) and w["q"].min() >= -32 and w["q"].max() <= 31
