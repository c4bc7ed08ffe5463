"""Parity of the W8A8 path (SmoothQuant factors, per-tensor INT8 / FP8 E4M3
quantization, the tcgen05 8-bit GEMM and the fused layer) with the oracle,
through the C ABI.

Quantization is integer/byte work: codes and scales bit-equal.  The INT8
layer accumulates exactly in int32 and applies the same fp32 epilogue as the
oracle, so its 16-bit outputs are bit-equal too.  The FP8 layer accumulates
in fp32 on the tensor cores where the oracle sums exactly; it is held to the
W4A16 tolerance (tests/helpers.py) against the oracle's exact product.
The GEMM is fed the oracle's own quantized operands, so no oracle input
comes from the CUDA path."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_pack_b200 as w4
from helpers import bits, check_y, odt

pytestmark = pytest.mark.gpu
DEV = "cuda"
FMTS = [(w4.W8_INT8, oracle.INT8), (w4.W8_E4M3, oracle.E4M3)]


def t_dtype(dtype):
    return torch.float16 if dtype == "f16" else torch.bfloat16


@pytest.mark.parametrize("fmt,ofmt", FMTS)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("op", [0, 1, 2])
@pytest.mark.parametrize("rows,K", [(1, 16), (7, 144), (300, 1024)])
def test_quantize_bit_exact(fmt, ofmt, dtype, op, rows, K):
    A = synth.activations(rows, K, rows + K + op, salient_frac=0.02, dtype=dtype)
    col = None
    if op:
        col = synth.activations(1, K, 77, dtype="f16")[0].float().abs().add(0.25)
    q, sc = w4.w8_quantize(A.to(DEV), fmt, None if col is None else col.to(DEV), op)
    torch.cuda.synchronize()
    qo, so = oracle.quant8(bits(A), odt(A), ofmt, None if col is None else col.numpy(), op)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert sc[0].item() == so


def test_quantize_zero_tensor():
    q, sc = w4.w8_quantize(torch.zeros(5, 64, dtype=torch.float16, device=DEV), w4.W8_INT8)
    torch.cuda.synchronize()
    assert sc[0].item() == 0.0 and int(q.count_nonzero()) == 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("alpha", [0.5, 0.25, 1.0])
def test_smooth_scales_bit_exact(dtype, alpha):
    X = synth.activations(40, 384, 3, salient_frac=0.02, dtype=dtype)
    W = synth.weights(300, 384, 0.02, 3, dtype=dtype)
    X[:, 11] = 0
    s = w4.w8_smooth_scales(X.to(DEV), W.to(DEV), alpha)
    torch.cuda.synchronize()
    so = oracle.smooth_scales(bits(X), bits(W), odt(X), float(np.float32(alpha)))
    assert np.array_equal(s.cpu().numpy(), so)


def oracle_operands(M, N, K, dtype, ofmt, seed, smooth=True):
    X = synth.activations(M, K, seed, salient_frac=0.01, dtype=dtype)
    W = synth.weights(N, K, 0.02, seed, dtype=dtype)
    s = oracle.smooth_scales(bits(X), bits(W), odt(X), 0.5) if smooth else None
    xq, sx = oracle.quant8(bits(X), odt(X), ofmt, s, 2 if smooth else 0)
    wq, sw = oracle.quant8(bits(W), odt(W), ofmt, s, 1 if smooth else 0)
    return X, W, s, xq, sx, wq, sw


def run_gemm(xq, sx, wq, sw, fmt, dtype):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    Y = w4.w8_gemm(dev(xq), dev(np.float32([sx])), dev(wq), dev(np.float32([sw])), fmt,
                   t_dtype(dtype))
    torch.cuda.synchronize()
    return Y


@pytest.mark.parametrize("fmt,ofmt", FMTS)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (33, 100, 144), (256, 128, 128), (300, 257, 512),
                                   (700, 520, 1024), (5, 3000, 2048)])
def test_gemm_parity(fmt, ofmt, dtype, M, N, K):
    X, W, s, xq, sx, wq, sw = oracle_operands(M, N, K, dtype, ofmt, M * 3 + N + K)
    Y = run_gemm(xq, sx, wq, sw, fmt, dtype)
    Yo = oracle.gemm8(xq, wq, ofmt, sx, sw, odt(X))
    if fmt == w4.W8_INT8:
        np.testing.assert_array_equal(Y.cpu().to(torch.float64).numpy(), Yo)
    else:
        check_y(Y, Yo, f"fp8 M={M} N={N} K={K}")
    assert w4.w4_device_status() == w4.W4_OK


@pytest.mark.parametrize("fmt,ofmt", FMTS)
def test_linear_end_to_end(fmt, ofmt):
    """w8a8_linear = quantize X / s on the fly + the 8-bit GEMM."""
    M, N, K = 200, 384, 768
    X, W, s, xq, sx, wq, sw = oracle_operands(M, N, K, "bf16", ofmt, 41)
    wqd = torch.from_numpy(wq).to(DEV)
    swd = torch.tensor([sw], dtype=torch.float32, device=DEV)
    Y = w4.w8a8_linear(X.to(DEV), wqd, swd, fmt, s=torch.from_numpy(s).to(DEV))
    torch.cuda.synchronize()
    Yo = oracle.gemm8(xq, wq, ofmt, sx, sw, oracle.BF16)
    if fmt == w4.W8_INT8:
        np.testing.assert_array_equal(Y.cpu().to(torch.float64).numpy(), Yo)
    else:
        check_y(Y, Yo, "fp8 linear")


def test_repeated_calls_identical():
    M, N, K = 512, 1024, 1024
    X, W, s, xq, sx, wq, sw = oracle_operands(M, N, K, "f16", oracle.E4M3, 5, smooth=False)
    a = run_gemm(xq, sx, wq, sw, w4.W8_E4M3, "f16")
    b = run_gemm(xq, sx, wq, sw, w4.W8_E4M3, "f16")
    assert torch.equal(a, b)


@pytest.mark.parametrize("fmt,ofmt", FMTS)
def test_full_size_sampled_rows(fmt, ofmt):
    """The W8A8 workload at full size (M = 2048, K = 4096, N = 11008, bf16,
    SmoothQuant alpha = 0.5 for INT8) through the device path end to end;
    192 sampled output rows checked against the oracle on the same inputs."""
    c = synth.W8A8
    M, K, N = c["M"], c["K"], c["N"]
    X = synth.activations(M, K, c["seed"], salient_frac=c["x_salient"], dtype=c["dtype"])
    W = synth.weights(N, K, c["std"], c["seed"], dtype=c["dtype"])
    smooth = fmt == w4.W8_INT8
    Xd, Wd = X.to(DEV), W.to(DEV)
    s = w4.w8_smooth_scales(Xd, Wd, c["alpha"]) if smooth else None
    wq, sw = w4.w8_quantize(Wd, fmt, s, w4.W8_COL_MUL if smooth else w4.W8_COL_NONE)
    Y = w4.w8a8_linear(Xd, wq, sw, fmt, s=s)
    torch.cuda.synchronize()
    so = oracle.smooth_scales(bits(X), bits(W), odt(X), c["alpha"]) if smooth else None
    xq, sxo = oracle.quant8(bits(X), odt(X), ofmt, so, 2 if smooth else 0)
    wqo, swo = oracle.quant8(bits(W), odt(W), ofmt, so, 1 if smooth else 0)
    assert np.array_equal(wq.cpu().numpy(), wqo) and sw[0].item() == swo
    rows = np.sort(np.random.default_rng(1).choice(M, 192, replace=False))
    Yo = oracle.gemm8(xq, wqo, ofmt, sxo, swo, odt(X), rows=rows)
    Ys = Y[torch.from_numpy(rows).to(DEV)]
    if fmt == w4.W8_INT8:
        np.testing.assert_array_equal(Ys.cpu().to(torch.float64).numpy(), Yo)
    else:
        check_y(Ys, Yo, "fp8 full size")
    assert w4.w4_device_status() == w4.W4_OK
