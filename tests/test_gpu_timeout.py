"""The give-up path of the kernels' bounded waits, driven on purpose (GPU only).

Every wait of the GEMV and GEMM kernels for another role or for data is bounded
(about 1 s by default).  qlinear_set_wait_limit shortens that bound to a few
hundred cycles and makes the producers withhold their copies (the flag that
nothing sets), so the first wait for data runs out: the kernel records the
time-out in the device status word, its roles leave their loops, tensor memory
is freed and the kernel returns.  Nothing faults or hangs.  The test checks that qlinear_sync_status reports QL_ERR_TIMEOUT,
and that the next call with the default bound returns QL_OK with the right
result, i.e. the context and the library stayed usable.
"""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from oracle import oracle_c as OC
from tests.gpu_helpers import Layer, assert_close, host, run_gemm, run_gemv, x_dev

pytestmark = pytest.mark.gpu

SHORT = 200  # cycles: far less than one copy from HBM takes


@pytest.mark.parametrize("fmt,fn,M", [("int4", "gemv", 1), ("int4", "gemv", 4), ("int6", "gemv", 2),
                                      ("int4", "gemm", 300), ("affine", "gemm", 256), ("affine", "gemm", 16)])
def test_short_wait_bound_times_out_then_recovers(cuda, fmt, fn, M):
    bits, group = (4, 64) if fmt == "affine" else (0, 0)
    L = Layer(fmt, 2048, 4096, seed=61, bits=bits, group=group)
    xb, xd = x_dev(4096, M, seed=62)
    call = ql.qlinear_gemv if fn == "gemv" else ql.qlinear_gemm
    assert ql.qlinear_sync_status() == ql.QL_OK  # nothing pending from earlier tests
    y = torch.empty((M, L.N), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_set_wait_limit(SHORT, withhold_copies=True)
    try:
        call(L.desc, *L.packed(), xd, M, y)
        status = ql.qlinear_sync_status()
    finally:
        ql.qlinear_set_wait_limit(0)  # back to the default bound, copies flowing
    assert status == ql.QL_ERR_TIMEOUT
    assert ql.qlinear_sync_status() == ql.QL_OK  # the status word was cleared by the read
    run = run_gemv if fn == "gemv" else run_gemm
    y_ok = run(L, xd, M)
    assert_close(y_ok, OC.matmul_f64(xb, L.oracle_w()), f"{fmt} {fn} M={M} after a time-out")
