"""Bias epilogue and N-concatenation of packed layers vs the oracle (GPU only)."""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from int6_quantized_linear_b200 import synth
from oracle import oracle_c as OC
from tests.gpu_helpers import Layer, assert_close, bf16_to_f64, dev, host, x_dev

pytestmark = pytest.mark.gpu


def bias_bits(N, seed):
    rng = np.random.default_rng(seed)
    return np.array([OC.bf16_from_f32(v) for v in rng.normal(0, 2.0, N).astype(np.float32)], np.uint16)


@pytest.mark.parametrize("fmt,bits,group,Ms", [("int4", 0, 0, (1, 3, 8)), ("int6", 0, 0, (1, 8)),
                                               ("affine", 4, 64, (1, 32))])
def test_gemv_bias(cuda, fmt, bits, group, Ms):
    N, K = 300, 2048
    L = Layer(fmt, N, K, seed=41, bits=bits, group=group)
    w_ref = L.oracle_w()
    bb = bias_bits(N, 42)
    bias = dev(bb).view(torch.bfloat16)
    for M in Ms:
        xb, xd = x_dev(K, M, seed=M + 7)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ql.qlinear_gemv_bias(L.desc, *L.packed(), xd, M, bias, y)
        assert ql.qlinear_sync_status() == ql.QL_OK
        y_ref = OC.matmul_f64(xb, w_ref) + bf16_to_f64(bb)[None, :]
        assert_close(host(y.view(torch.int16), np.uint16), y_ref, f"gemv bias {fmt} M={M}")


@pytest.mark.parametrize("fmt,bits,group", [("int4", 0, 0), ("affine", 8, 128)])
def test_gemm_bias(cuda, fmt, bits, group):
    N, K, M = 1000, 1024, 300
    L = Layer(fmt, N, K, seed=43, bits=bits, group=group)
    w_ref = L.oracle_w()
    bb = bias_bits(N, 44)
    xb, xd = x_dev(K, M, seed=45)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_gemm_bias(L.desc, *L.packed(), xd, M, dev(bb).view(torch.bfloat16), y)
    assert ql.qlinear_sync_status() == ql.QL_OK
    y_ref = OC.matmul_f64(xb, w_ref) + bf16_to_f64(bb)[None, :]
    assert_close(host(y.view(torch.int16), np.uint16), y_ref, f"gemm bias {fmt}")


def test_bias_entry_points_need_a_bias(cuda):
    L = Layer("int4", 64, 256, seed=1)
    xd = x_dev(256, 1, 1)[1]
    y = torch.empty((1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_gemv_bias(L.desc, *L.packed(), xd, 1, None, y)
    assert e.value.status == ql.QL_ERR_NULL


@pytest.mark.parametrize("fmt,bits,group", [("int4", 0, 0), ("int6", 0, 0), ("affine", 2, 64)])
def test_concat_n(cuda, fmt, bits, group):
    """Stacking two packed layers along N equals packing the stacked inputs (bit-exact), and the
    stacked layer's GEMV equals the oracle on the stacked weights."""
    K = 1024
    A = Layer(fmt, 300, K, seed=51, bits=bits, group=group)
    B = Layer(fmt, 513, K, seed=52, bits=bits, group=group)
    stacked = {k: np.concatenate([A.w[k], B.w[k]], 0) for k in A.w}
    C = Layer(fmt, 813, K, seed=0, bits=bits, group=group, weights=stacked)
    out = ql.alloc_packed(C.desc)
    ql.qlinear_concat_n(A.desc, A.packed(), B.desc, B.packed(), out)
    assert ql.qlinear_sync_status() == ql.QL_OK
    nc, ng, ns = ql.qlinear_packed_bytes(C.desc)
    for got, want, n in zip(out, C.packed(), (nc, ng, ns)):
        if n:
            assert np.array_equal(host(got, np.uint8)[:n], host(want, np.uint8)[:n])
    xb, xd = x_dev(K, 1, seed=53)
    y = torch.empty((1, 813), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_gemv(C.desc, *out, xd, 1, y)
    assert ql.qlinear_sync_status() == ql.QL_OK
    assert_close(host(y.view(torch.int16), np.uint16), OC.matmul_f64(xb, np.concatenate([A.oracle_w(), B.oracle_w()])),
                 f"concat gemv {fmt}")


def test_concat_rejects_mismatched_layers(cuda):
    A = Layer("int4", 64, 256, seed=1)
    B = Layer("int4", 64, 512, seed=2)
    out = ql.alloc_packed(ql.Desc("int4", 128, 256))
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_concat_n(A.desc, A.packed(), B.desc, B.packed(), out)
    assert e.value.status == ql.QL_ERR_SHAPE
