"""qlinear_gemm_noalloc: the GEMM for callers that may not allocate device memory.

Such callers (an op behind a runtime's plug-in interface that only hands over
input and output pointers, or a process that has reserved all of HBM for its
own pool) cannot provide qlinear_gemm's workspace; this entry point takes it
from a fixed device array inside the library instead.  The test calls it
several times in a row through the C ABI, on different layers (int4, int6 and
2-bit affine, the last with N not a multiple of 32 so that padded weight rows
meet whatever the previous call left in the shared array), and checks each
result bit for bit against qlinear_gemm's on the same inputs (both run the
same kernels) and against the oracle within the tolerance the parity tests
use.  The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from oracle import oracle_c as OC
from tests.gpu_helpers import Layer, assert_close, host, run_gemm, x_dev

pytestmark = pytest.mark.gpu


def test_gemm_noalloc_matches_gemm_in_a_row(cuda):
    cases = (("int4", 1000, 1024, 200, 11, 0, 0), ("int6", 300, 2048, 70, 12, 0, 0),
             ("affine", 333, 1024, 150, 14, 2, 64), ("int4", 97, 512, 300, 15, 0, 0))
    for fmt, N, K, M, seed, bits, group in cases:
        L = Layer(fmt, N, K, seed, bits, group)
        xb, xd = x_dev(K, M, seed)
        y_ref = run_gemm(L, xd, M)  # the existing entry point, with its own workspace
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ql.qlinear_gemm_noalloc(L.desc, *L.packed(), xd, M, y)
        assert ql.qlinear_sync_status() == ql.QL_OK
        got = host(y.view(torch.int16), np.uint16)
        assert np.array_equal(got, y_ref), f"noalloc {fmt} N={N} M={M} differs from qlinear_gemm"
        assert_close(got, OC.matmul_f64(xb, L.oracle_w()), f"noalloc {fmt} N={N} M={M}")


def test_gemm_noalloc_rejects_problems_beyond_its_scratch(cuda):
    L = Layer("int4", 256, 4096, seed=13)
    M = 4096  # needs 2*M*K = 32 MiB for x alone, plus the scales
    assert ql.qlinear_gemm_workspace_bytes(L.desc, M) > 32 * 1024 * 1024
    x = torch.zeros((M, 4096), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_gemm_noalloc(L.desc, *L.packed(), x, M, y)
    assert e.value.status == ql.QL_ERR_RANGE
    assert ql.qlinear_sync_status() == ql.QL_OK
