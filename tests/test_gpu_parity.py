"""CUDA path vs the CPU oracle, through the C ABI (GPU only).

Bit-exact: pack, unpack, fp32 dequant, bf16 dequant.  Within the stated
tolerance (see gpu_helpers.assert_close): the GEMV and the tcgen05 GEMM.
Small shapes are compared element by element; the full layer shapes are
compared on sampled output rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import int6_quantized_linear_b200 as ql
from int6_quantized_linear_b200 import synth
from oracle import oracle_c as OC
from oracle import oracle_np as ON
from tests.gpu_helpers import Layer, assert_close, bf16_to_f64, dev, host, run_gemm, run_gemv, x_dev

pytestmark = pytest.mark.gpu

FORMATS = [("int4", 0, 0), ("int6", 0, 0), ("int6p", 0, 0), ("affine", 2, 64), ("affine", 4, 64),
           ("affine", 8, 64), ("affine", 4, 32), ("affine", 8, 128)]
FMT_IDS = [f"{f}{b or ''}g{g or ''}" for f, b, g in FORMATS]
# several tiles plus a ragged tail in N; K of one super-block and several
SMALL_SHAPES = [(1, 256), (7, 512), (33, 1024), (300, 2048), (513, 768)]


@pytest.mark.parametrize("fmt,bits,group", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
def test_pack_unpack_dequant_bitexact(cuda, fmt, bits, group, N, K):
    L = Layer(fmt, N, K, seed=N + K, bits=bits, group=group)
    got = L.packed_host()
    want = L.oracle_pack()
    for a, b in zip(got, want):
        if b is not None:
            assert np.array_equal(a, b)
    # unpack on the GPU recovers the inputs
    u = L.unpacked_host()
    outs = [torch.empty_like(dev(a)) if a is not None else None for a in u]
    ql.qlinear_unpack(L.desc, *L.packed(), *outs)
    for a, o in zip(u, outs):
        if a is not None:
            assert np.array_equal(host(o, a.dtype).reshape(a.shape), a)
    # dequant, fp32 bit-exact and bf16 = nearest-even of the fp32 value
    w_ref = L.oracle_w()
    w32 = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ql.qlinear_dequant(L.desc, *L.packed(), w32, ql.QL_OUT_F32)
    assert np.array_equal(host(w32, np.uint32), w_ref.view(np.uint32))
    w16 = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_dequant(L.desc, *L.packed(), w16, ql.QL_OUT_BF16)
    got16 = host(w16.view(torch.int16), np.uint16).reshape(N, K)
    assert np.array_equal(got16, ON.bf16_bits_from_f32(w_ref))  # every element
    want16 = np.array([OC.bf16_from_f32(v) for v in w_ref.ravel()[:4096]], np.uint16)  # C oracle's rounding
    assert np.array_equal(got16.ravel()[:4096], want16)
    assert ql.qlinear_sync_status() == ql.QL_OK


@pytest.mark.parametrize("fmt,bits,group", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
def test_gemv_small(cuda, fmt, bits, group, N, K):
    L = Layer(fmt, N, K, seed=3 * N + K, bits=bits, group=group)
    w_ref = L.oracle_w()
    for M in ((1, 2, 3, 5, 8) if fmt != "affine" else (1, 4, 8, 13, 32)):
        xb, xd = x_dev(K, M, seed=M)
        y = run_gemv(L, xd, M)
        assert_close(y, OC.matmul_f64(xb, w_ref), f"gemv {fmt} N={N} K={K} M={M}")


@pytest.mark.parametrize("fmt,bits,group", [("int4", 0, 0), ("int6", 0, 0), ("int6p", 0, 0), ("affine", 4, 64),
                                            ("affine", 2, 32), ("affine", 8, 128)])
@pytest.mark.parametrize("N,K,Ms", [(256, 256, (1, 127, 128)), (300, 512, (129, 200)),
                                    (1000, 1024, (64, 256)), (40, 768, (300,))])
def test_gemm_small(cuda, fmt, bits, group, N, K, Ms):
    L = Layer(fmt, N, K, seed=N + 5 * K, bits=bits, group=group)
    w_ref = L.oracle_w()
    for M in Ms:
        xb, xd = x_dev(K, M, seed=M + 1)
        y = run_gemm(L, xd, M)
        assert_close(y, OC.matmul_f64(xb, w_ref), f"gemm {fmt} N={N} K={K} M={M}")


def _sampled_rows(N, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(count, N), replace=False)]))
    return rows


@pytest.mark.parametrize("name", ["int4_gemv_2048x2048", "int4_gemv_k5120_n27648", "int4_gemv_k27648_n5120",
                                  "int6_gemv_k5120_n5120", "int6_gemv_k5120_n27648",
                                  "int6p_gemv_k5120_n5120", "int6p_gemv_k5120_n27648",
                                  "affine2_k4096_n14336", "affine4_k4096_n14336", "affine8_k4096_n14336"])
def test_gemv_full_size_sampled(cuda, name):
    wl = synth.WORKLOADS[name]
    L = Layer(wl.fmt, wl.N, wl.K, wl.seed, wl.bits, wl.group)
    # packed bytes of the full layer are bit-exact
    got = L.packed_host()
    want = L.oracle_pack()
    for a, b in zip(got, want):
        if b is not None:
            assert np.array_equal(a, b)
    rows = _sampled_rows(wl.N, 384, wl.seed)
    w_ref = L.oracle_w(rows)
    xb8 = wl.x(max(wl.Ms))
    for M in wl.Ms:
        xd = dev(xb8[:M])
        y = run_gemv(L, xd, M)
        y_ref = OC.matmul_f64(xb8[:M], w_ref)
        assert_close(y[:, rows], y_ref, f"gemv {name} M={M}")


@pytest.mark.parametrize("N,K", [(14400, 6144), (16384, 11520), (5000, 256)])
def test_gemv_int4_m1_part_sizes(cuda, N, K):
    """int4 at M=1 where the parts of K are set by how much x a CTA holds (at most 22 super-blocks):
    K = 6144 and 11520 with enough rows to fill every CTA slot unsplit still split K in two and
    three parts; K = 256 is a single super-block.  Sampled rows (all of them for the last case)
    checked against the oracle, bits repeatable."""
    L = Layer("int4", N, K, seed=N + K)
    rows = _sampled_rows(N, 384, N) if N * K > 4_000_000 else np.arange(N)
    w_ref = L.oracle_w(rows)
    xb, xd = x_dev(K, 1, seed=K + 5)
    y = run_gemv(L, xd, 1)
    assert_close(y[:, rows], OC.matmul_f64(xb, w_ref), f"int4 M=1 N={N} K={K}")
    assert np.array_equal(y, run_gemv(L, xd, 1))


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_gemm_full_size_sampled(cuda, M):
    wl = synth.WORKLOADS["int4_gemm_k5120_n27648"]
    L = Layer(wl.fmt, wl.N, wl.K, wl.seed)
    rows = _sampled_rows(wl.N, 192, M)
    w_ref = L.oracle_w(rows)
    xb = wl.x(M)
    y = run_gemm(L, dev(xb), M)
    toks = _sampled_rows(M, 96, M + 1)
    y_ref = OC.matmul_f64(xb[toks], w_ref)
    assert_close(y[np.ix_(toks, rows)], y_ref, f"gemm full M={M}")


@pytest.mark.parametrize("fmt,bits,group", [("int4", 0, 0), ("int6", 0, 0), ("affine", 4, 64)])
@pytest.mark.parametrize("M", [24, 600])
def test_gemm_ragged_multi_tile(cuda, fmt, bits, group, M):
    """Several tiles per CTA in both GEMM forms, with a ragged last row tile (N = 20000 = 156 x 128 +
    32): M = 24 runs the 32-token form (157 tiles, so some CTAs use both accumulators in turn), M = 600
    the 256-token form (3 x 157 tiles, the last token tile 88 tokens: the accumulator is handed from
    tile to tile).  Sampled rows (the last 40 included) and tokens against the oracle; a second call
    must give the same bits."""
    N, K = 20000, 1024
    L = Layer(fmt, N, K, seed=7 * M + K, bits=bits, group=group)
    rows = np.unique(np.concatenate([_sampled_rows(N, 160, M), np.arange(N - 40, N)]))
    w_ref = L.oracle_w(rows)
    xb, xd = x_dev(K, M, seed=M + 11)
    y = run_gemm(L, xd, M)
    toks = _sampled_rows(M, 48, M + 3)
    assert_close(y[np.ix_(toks, rows)], OC.matmul_f64(xb[toks], w_ref), f"gemm {fmt} N={N} K={K} M={M}")
    assert np.array_equal(y, run_gemm(L, xd, M))


def test_gemm_error_budget(cuda):
    """fp16 operands with per-row power-of-two scales: the only rounding beyond fp32 accumulation is
    one 11-bit rounding per weight, so the error stays far inside the gate (bf16 weights would use ~100%)."""
    L = Layer("int4", 1024, 2048, seed=77)
    w_ref = L.oracle_w()
    xb, xd = x_dev(2048, 256, seed=9)
    y = run_gemm(L, xd, 256)
    used = assert_close(y, OC.matmul_f64(xb, w_ref), "gemm budget")
    assert used < 3e-3, used


def test_deterministic_and_in_bounds(cuda):
    """Two runs give identical bits (including the M=1 GEMV, whose tiles are split between warps
    and added up by whichever warp finishes a tile last); sentinel bytes around the output are untouched."""
    L = Layer("int4", 1000, 2048, seed=5)
    for runner, M in ((run_gemv, 3), (run_gemv, 1), (run_gemm, 200)):
        xb, xd = x_dev(2048, M, seed=2)
        pad = 4096
        buf = torch.full((pad + M * 1000 + pad,), 0x7B7B, dtype=torch.int16, device="cuda")
        y = buf[pad:pad + M * 1000].view(torch.bfloat16).view(M, 1000)
        fn = ql.qlinear_gemv if runner is run_gemv else ql.qlinear_gemm
        fn(L.desc, *L.packed(), xd, M, y)
        first = host(y.view(torch.int16).clone(), np.uint16)
        fn(L.desc, *L.packed(), xd, M, y)
        assert ql.qlinear_sync_status() == ql.QL_OK
        assert np.array_equal(first, host(y.view(torch.int16), np.uint16))
        b = host(buf, np.uint16)
        assert np.all(b[:pad] == 0x7B7B) and np.all(b[pad + M * 1000:] == 0x7B7B)


@pytest.mark.parametrize("bits,group", [(2, 64), (2, 32)])
@pytest.mark.parametrize("N,K", [(200, 1536), (64, 256), (700, 4096)])
def test_gemv_affine2_multi_token(cuda, bits, group, N, K):
    """2-bit affine on the multi-token tensor-core GEMV (64-byte swizzled code rows) at M = 1..8,
    with and without the K split; repeated runs give identical bits."""
    L = Layer("affine", N, K, seed=13 * N + K + group, bits=bits, group=group)
    w_ref = L.oracle_w()
    for M in range(1, 9):
        xb, xd = x_dev(K, M, seed=200 + M)
        y = run_gemv(L, xd, M)
        assert_close(y, OC.matmul_f64(xb, w_ref), f"affine{bits} g{group} gemv N={N} K={K} M={M}")
        assert np.array_equal(y, run_gemv(L, xd, M))


@pytest.mark.parametrize("bits,group", [(2, 64), (4, 64), (8, 64), (2, 32), (4, 32), (8, 32)])
@pytest.mark.parametrize("N,K", [(200, 1536), (64, 256), (1000, 4096)])
def test_gemv_affine_f16_token_counts(cuda, bits, group, N, K):
    """Affine at 9..32 tokens on the fp16 tensor-core GEMV (two or four 8-token column tiles, K split
    over CTAs for the small layers, ragged N): every token count on its own layer checked against the
    oracle; repeated runs give identical bits; the bias variant adds bias[n]."""
    L = Layer("affine", N, K, seed=17 * N + K + bits, bits=bits, group=group)
    w_ref = L.oracle_w()
    bias_b = synth.activations(N + 3 * K, 1, N)[0]
    xb32, _ = x_dev(K, 32, seed=300 + bits)
    for M in (9, 10, 15, 16, 17, 23, 24, 31, 32):
        xb = xb32[:M]
        xd = dev(xb)
        y = run_gemv(L, xd, M)
        y_ref = OC.matmul_f64(xb, w_ref)
        assert_close(y, y_ref, f"affine{bits} g{group} f16 gemv N={N} K={K} M={M}")
        assert np.array_equal(y, run_gemv(L, xd, M))
        if M in (9, 32):
            yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            ql.qlinear_gemv_bias(L.desc, *L.packed(), xd, M, dev(bias_b).view(torch.bfloat16), yb)
            assert ql.qlinear_sync_status() == ql.QL_OK
            assert_close(host(yb.view(torch.int16), np.uint16), y_ref + bf16_to_f64(bias_b)[None, :],
                         f"affine{bits} g{group} f16 gemv+bias M={M}")


@pytest.mark.parametrize("bits,group", [(4, 64), (2, 32), (8, 64)])
@pytest.mark.parametrize("N,K", [(37900, 512), (3000, 2304)])
def test_gemv_affine_f16_unit_ranges(cuda, bits, group, N, K):
    """The fp16 GEMV on larger layers: K = 512 with far more 64-row groups than CTA slots and a ragged
    last group, K = 2304 with its K split over CTAs; every output checked against the oracle, bits
    repeatable."""
    L = Layer("affine", N, K, seed=19 * N + K + bits, bits=bits, group=group)
    w_ref = L.oracle_w()
    xb32, _ = x_dev(K, 32, seed=400 + bits)
    for M in (9, 32):
        xb = xb32[:M]
        xd = dev(xb)
        y = run_gemv(L, xd, M)
        assert_close(y, OC.matmul_f64(xb, w_ref), f"affine{bits} g{group} f16 gemv N={N} K={K} M={M}")
        assert np.array_equal(y, run_gemv(L, xd, M))


@pytest.mark.parametrize("fmt", ["int6", "int6p"])
@pytest.mark.parametrize("N,K", [(200, 1536), (64, 256), (1000, 5120)])
def test_gemv_int6_every_token_count(cuda, fmt, N, K):
    """int6 tensor-core GEMV (dense and planar storage) at each M it serves (1..8: four token
    buckets), with and without the split of K over CTAs; repeated runs give identical bits; the bias
    variant adds bias[n]."""
    L = Layer(fmt, N, K, seed=11 * N + K)
    w_ref = L.oracle_w()
    bias_b = synth.activations(N + K, 1, N)[0]
    for M in range(1, 9):
        xb, xd = x_dev(K, M, seed=100 + M)
        y = run_gemv(L, xd, M)
        y_ref = OC.matmul_f64(xb, w_ref)
        assert_close(y, y_ref, f"{fmt} gemv N={N} K={K} M={M}")
        assert np.array_equal(y, run_gemv(L, xd, M))
        yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ql.qlinear_gemv_bias(L.desc, *L.packed(), xd, M, dev(bias_b).view(torch.bfloat16), yb)
        assert ql.qlinear_sync_status() == ql.QL_OK
        assert_close(host(yb.view(torch.int16), np.uint16), y_ref + bf16_to_f64(bias_b)[None, :],
                     f"int6 gemv+bias M={M}")


def test_device_errors_do_not_launch(cuda):
    L = Layer("int4", 64, 256, seed=1)
    xd = x_dev(256, 1, 1)[1]
    y = torch.empty((1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_gemv(L.desc, *L.packed(), xd, 9, y)
    assert e.value.status == ql.QL_ERR_RANGE
    with pytest.raises(ql.QLinearError) as e:
        ql.qlinear_gemv(L.desc, L.codes[1:], L.gmeta, L.steps, xd, 1, y)
    assert e.value.status == ql.QL_ERR_ALIGN
    assert ql.qlinear_sync_status() == ql.QL_OK
