"""The metadata encoder on the GPU vs the oracle (bit-exact codes and steps), its domain check,
and its end-to-end effect on the weights (GPU only)."""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from oracle import oracle_np as O
from tests.gpu_helpers import host

pytestmark = pytest.mark.gpu


def int4_fields(N, K, seed):
    rng = np.random.default_rng(seed)
    G = K // 32
    scale = rng.uniform(1e-4, 1e-2, (N, G)).astype(np.float32)
    zero = (rng.uniform(0, 15, (N, G)) * (rng.random((N, G)) > 0.1)).astype(np.float32)
    zero[0, :8] = 0.0  # a super-block of zero points that are all 0
    scale[-1, -8:] = np.float32(2.0 ** -20)  # tiny steps (fp16 subnormal after / 255)
    return scale, zero


def run_int4(scale, zero):
    N, G = scale.shape
    d = ql.Desc("int4", N, 32 * G)
    dev = lambda a: torch.from_numpy(a).cuda()
    sc = torch.empty((N, G), dtype=torch.uint8, device="cuda")
    zc = torch.empty_like(sc)
    ss = torch.empty((N, G // 8), dtype=torch.int16, device="cuda")
    zs = torch.empty_like(ss)
    ql.qlinear_quantize_meta(d, dev(scale), dev(zero), sc, zc, ss, zs)
    st = ql.qlinear_sync_status()
    return st, host(sc, np.uint8), host(zc, np.uint8), host(ss, np.uint16), host(zs, np.uint16)


@pytest.mark.parametrize("N,K", [(1, 256), (300, 2048), (27648, 5120)])
def test_int4_encoder_bitexact(cuda, N, K):
    scale, zero = int4_fields(N, K, seed=N + K)
    st, sc, zc, ss, zs = run_int4(scale, zero)
    assert st == ql.QL_OK
    esc, ess = O.encode_u8_per_super(scale, 8)
    ezc, ezs = O.encode_u8_per_super(zero, 8)
    assert np.array_equal(sc, esc) and np.array_equal(ss, ess)
    assert np.array_equal(zc, ezc) and np.array_equal(zs, ezs)


@pytest.mark.parametrize("N,K", [(3, 256), (513, 4096)])
def test_int6_encoder_bitexact(cuda, N, K):
    rng = np.random.default_rng(K)
    G = K // 16
    scale = (rng.uniform(1e-4, 1e-2, (N, G)) * rng.choice([-1, 1], (N, G))).astype(np.float32)
    scale[0, :16] = 0.0
    d = ql.Desc("int6", N, K)
    sc = torch.empty((N, G), dtype=torch.int8, device="cuda")
    st = torch.empty((N, K // 256), dtype=torch.int16, device="cuda")
    ql.qlinear_quantize_meta(d, torch.from_numpy(scale).cuda(), None, sc, None, st, None)
    assert ql.qlinear_sync_status() == ql.QL_OK
    esc, est = O.encode_i8_per_super(scale, 16)
    assert np.array_equal(host(sc, np.int8), esc)
    assert np.array_equal(host(st, np.uint16), est)


def test_encoder_domain_is_checked(cuda):
    scale, zero = int4_fields(8, 512, seed=3)
    zero[5, 7] = -0.25  # a negative zero point: the encoder must not silently clamp it
    st, *_ = run_int4(scale, zero)
    assert st == ql.QL_ERR_RANGE
    scale[2, 2] = np.nan
    st, *_ = run_int4(scale, np.abs(zero))
    assert st == ql.QL_ERR_RANGE
    st, *_ = run_int4(np.abs(np.nan_to_num(scale)), np.abs(zero))
    assert st == ql.QL_OK  # the status word was cleared by the previous read


def test_encoder_end_to_end_snr(cuda):
    """Encode float metadata on the GPU, pack with random codes, dequantise on the GPU; the weights
    differ from those of the float metadata only by the half-step code rounding (SNR well above
    the 4-bit codes' own noise floor)."""
    N, K = 256, 2048
    scale, zero = int4_fields(N, K, seed=11)
    st, sc, zc, ss, zs = run_int4(scale, zero)
    assert st == ql.QL_OK
    rng = np.random.default_rng(12)
    q = rng.integers(0, 16, (N, K), dtype=np.uint8)
    d = ql.Desc("int4", N, K)
    c, g, s = ql.alloc_packed(d, "cuda")
    t = lambda a: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()
    ql.qlinear_pack(d, t(q), t(sc), t(zc), t(ss), t(zs), c, g, s)
    w = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ql.qlinear_dequant(d, c, g, s, w, ql.QL_OUT_F32)
    assert ql.qlinear_sync_status() == ql.QL_OK
    w_float = (q.astype(np.float64) - np.repeat(zero, 32, 1)) * np.repeat(scale, 32, 1)
    snr = O.snr_db(w_float, host(w, np.float32))
    assert snr > 40.0, snr
