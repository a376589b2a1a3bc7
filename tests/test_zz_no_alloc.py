"""qlinear_gemm_noalloc: the GEMM for callers that may not allocate device memory.

Such callers (an op behind a runtime's plug-in interface that only hands over
input and output pointers, or a process that has reserved all of HBM for its
own pool) cannot provide qlinear_gemm's workspace; this entry point takes it
from a fixed device array inside the library instead.  The test calls it
twice in a row through the C ABI, on different layers, and checks each result
against qlinear_gemm's within the tolerance the parity tests use.  The file
name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from tests.gpu_helpers import Layer, assert_close, bf16_to_f64, host, run_gemm, x_dev

pytestmark = pytest.mark.gpu


def test_gemm_noalloc_matches_gemm_twice(cuda):
    for fmt, N, K, M, seed in (("int4", 1000, 1024, 200, 11), ("int6", 300, 2048, 70, 12)):
        L = Layer(fmt, N, K, seed)
        xb, xd = x_dev(K, M, seed)
        y_ref = run_gemm(L, xd, M)  # the existing entry point, with its own workspace
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ql.qlinear_gemm_noalloc(L.desc, *L.packed(), xd, M, y)
        assert ql.qlinear_sync_status() == ql.QL_OK
        assert_close(host(y.view(torch.int16), np.uint16), bf16_to_f64(y_ref), f"noalloc {fmt} M={M}")


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
