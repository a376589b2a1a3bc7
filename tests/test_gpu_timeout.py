"""The give-up path of the kernels' bounded waits, driven on purpose (GPU only).

Every wait of the GEMV and GEMM kernels for another role or for data is bounded
(2e9 SM cycles, about 1 s).  qlinear_set_withhold_copies makes the producers
start no copies (the flag that nothing sets), so the first wait for data runs
out after that second: the kernel records the time-out in the device status
word, its roles leave their loops, tensor memory is freed and the kernel
returns.  Nothing faults or hangs.  The test checks that qlinear_sync_status
reports QL_ERR_TIMEOUT, and that the next call, with copies flowing, returns
QL_OK with the right result, i.e. the context and the library stayed usable.
"""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from oracle import oracle_c as OC
from tests.gpu_helpers import Layer, assert_close, host, run_gemm, run_gemv, x_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,fn,M", [("int4", "gemv", 1), ("int4", "gemv", 4), ("int6", "gemv", 2),
                                      ("int4", "gemm", 300), ("affine", "gemm", 256), ("affine", "gemm", 16)])
def test_wait_runs_out_then_recovers(cuda, fmt, fn, M):
    bits, group = (4, 64) if fmt == "affine" else (0, 0)
    L = Layer(fmt, 2048, 4096, seed=61, bits=bits, group=group)
    xb, xd = x_dev(4096, M, seed=62)
    call = ql.qlinear_gemv if fn == "gemv" else ql.qlinear_gemm
    assert ql.qlinear_sync_status() == ql.QL_OK  # nothing pending from earlier tests
    y = torch.empty((M, L.N), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_set_withhold_copies(True)
    try:
        call(L.desc, *L.packed(), xd, M, y)
        status = ql.qlinear_sync_status()  # about 1 s: the first wait for data runs out
    finally:
        ql.qlinear_set_withhold_copies(False)  # copies flowing again
    assert status == ql.QL_ERR_TIMEOUT
    assert ql.qlinear_sync_status() == ql.QL_OK  # the status word was cleared by the read
    run = run_gemv if fn == "gemv" else run_gemm
    y_ok = run(L, xd, M)
    assert_close(y_ok, OC.matmul_f64(xb, L.oracle_w()), f"{fmt} {fn} M={M} after a time-out")
