"""Pins of the oracle's W8A8 functions (SmoothQuant factors, per-tensor INT8
and FP8 E4M3 quantization, the 8-bit layer) to facts that do not come from
the oracle itself.

Sources: "LLM quantization methods: principles and implementation" §2.2
(symmetric INT8: scale = max|x| / 127, round, clamp), §4.3 (SmoothQuant:
s_j = max|X_j|^alpha / max|W_j|^(1-alpha), X' = X / s, W' = W * s, both INT8
per tensor) and §4.6 (FP8 E4M3: scale = max|x| / 448, cast).
The pins: the E4M3 codec against torch's float8_e4m3fn for every code and
for random values; INT8 codes against numpy rounding where the scale is 1;
the factors against numpy column maxima; the identity X'W'^T = XW^T exactly
when s is a power of two; the integer accumulation against numpy's int64
matmul; the FP8 product against numpy's fp64 matmul; and the method's claim
that smoothing cuts the W8A8 error on activations with outlier channels.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def vals(t):
    return t.to(torch.float64).numpy()


def test_e4m3_decode_every_code():
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_e4m3_rounding_against_torch():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(4000) * 10.0 ** rng.integers(-4, 3, 4000)).astype(np.float32)
    v = np.concatenate([v[np.abs(v) <= 448], np.float32([448, -448, 0.0, 2.0 ** -10, 3 * 2.0 ** -11,
                                                          0.0625 + 2.0 ** -8, 15.5, 464.0 - 1e-3])])
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.round_e4m3(float(x)) for x in v])
    np.testing.assert_array_equal(got, want)
    assert oracle.round_e4m3(1000.0) == 448.0 and oracle.round_e4m3(-500.0) == -448.0


def test_int8_unit_scale_is_numpy_round():
    x = np.concatenate([[127.0, -126.5, 2.5, 3.5, -0.5, 0.49], np.linspace(-120, 120, 250)])
    A = torch.from_numpy(x.reshape(2, -1)).to(torch.float16)
    q, sc = oracle.quant8(bits(A), oracle.F16, oracle.INT8)
    assert sc == np.float32(1.0)
    want = np.clip(np.round(vals(A)), -127, 127).astype(np.int8)
    np.testing.assert_array_equal(q.view(np.int8), want)


@pytest.mark.parametrize("fmt", [oracle.INT8, oracle.E4M3])
def test_quant8_codes_against_library(fmt):
    A = synth.activations(16, 256, 4, salient_frac=0.02)
    col = np.float32(2.0) ** np.random.default_rng(4).integers(-3, 4, 256).astype(np.float32)
    for op in (0, 1, 2):
        q, sc = oracle.quant8(bits(A), oracle.F16, fmt, col if op else None, op)
        v = vals(A).astype(np.float32)
        v = v * col if op == 1 else (v / col if op == 2 else v)
        qmax = np.float32(127.0 if fmt == oracle.INT8 else 448.0)
        assert sc == np.abs(v).max() / qmax
        t = v / sc
        if fmt == oracle.INT8:
            np.testing.assert_array_equal(q.view(np.int8), np.clip(np.round(t), -127, 127))
        else:
            want = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            np.testing.assert_array_equal(q, want)


def test_zero_tensor_quantizes_to_zero():
    q, sc = oracle.quant8(np.zeros((3, 64), np.uint16), oracle.F16, oracle.INT8)
    assert sc == 0.0 and not q.any()


def test_smooth_scales_against_numpy():
    X = synth.activations(32, 384, 5, salient_frac=0.02)
    W = synth.weights(48, 384, 0.02, 5)
    X[:, 7] = 0.0
    for alpha in (0.5, 0.8):
        s = oracle.smooth_scales(bits(X), bits(W), oracle.F16, alpha)
        a = np.abs(vals(X)).max(0)
        w = np.abs(vals(W)).max(0)
        with np.errstate(divide="ignore", invalid="ignore"):
            want = (np.power(a, alpha).astype(np.float32) /
                    np.power(w, 1 - alpha).astype(np.float32))
        want = np.maximum(want, np.float32(1e-5))
        want[7] = 1.0
        np.testing.assert_array_equal(s, want)


def test_smoothing_is_an_identity_for_power_of_two_factors():
    """max|X_j| = 4^e_j and max|W_j| = 1 give s_j = 2^e_j at alpha = 0.5; then
    fl(X / s) and fl(W * s) are exact and X' W'^T = X W^T exactly."""
    rng = np.random.default_rng(6)
    K = 256
    e = rng.integers(-2, 3, K)
    X = rng.integers(-60, 61, (8, K)).astype(np.float64) / 64 * 4.0 ** e
    X[0] = 4.0 ** e
    W = rng.integers(-100, 101, (16, K)).astype(np.float64) / 128
    W[0] = 1.0
    Xt = torch.from_numpy(X).to(torch.float16)
    Wt = torch.from_numpy(W).to(torch.float16)
    s = oracle.smooth_scales(bits(Xt), bits(Wt), oracle.F16, 0.5)
    np.testing.assert_array_equal(s, (2.0 ** e).astype(np.float32))
    Xs = vals(Xt) / s
    Ws = vals(Wt) * s
    np.testing.assert_array_equal(Xs @ Ws.T, vals(Xt) @ vals(Wt).T)


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_int8_layer_against_numpy(dtype):
    rng = np.random.default_rng(7)
    # 64 x 512 outputs: enough that an fp64 epilogue would round a few fp16
    # outputs differently from the fp32 one (3 of them for this seed)
    Xq = rng.integers(-127, 128, (64, 1024)).astype(np.int8)
    Wq = rng.integers(-127, 128, (512, 1024)).astype(np.int8)
    sx, sw = np.float32(0.0123), np.float32(0.00071)
    Y = oracle.gemm8(Xq.view(np.uint8), Wq.view(np.uint8), oracle.INT8, sx, sw, dtype)
    acc = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    y = acc.astype(np.float32) * np.float32(sx * sw)
    if dtype == oracle.F16:
        want = y.astype(np.float16).astype(np.float64)
    else:
        want = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(Y, want)
    rows = np.array([63, 0, 3])
    np.testing.assert_array_equal(
        oracle.gemm8(Xq.view(np.uint8), Wq.view(np.uint8), oracle.INT8, sx, sw, dtype, rows=rows),
        Y[rows])


def test_fp8_layer_against_numpy():
    rng = np.random.default_rng(8)
    Xq = rng.integers(0, 256, (7, 384)).astype(np.uint8)
    Wq = rng.integers(0, 256, (21, 384)).astype(np.uint8)
    Xq[(Xq & 0x7F) == 0x7F] = 0  # no NaN codes
    Wq[(Wq & 0x7F) == 0x7F] = 0
    sx, sw = np.float32(0.02), np.float32(0.5)
    Y = oracle.gemm8(Xq, Wq, oracle.E4M3, sx, sw, oracle.BF16)
    dec = lambda q: torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    want = dec(Xq) @ dec(Wq).T * np.float64(sx) * np.float64(sw)
    np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-12)


def w8a8_error(X, W, fmt, s=None):
    """Relative Frobenius error of the quantized layer against X W^T."""
    xq, sx = oracle.quant8(bits(X), oracle.F16, fmt, s, 2 if s is not None else 0)
    wq, sw = oracle.quant8(bits(W), oracle.F16, fmt, s, 1 if s is not None else 0)
    Y = oracle.gemm8(xq, wq, fmt, sx, sw, oracle.F16)
    ref = vals(X) @ vals(W).T
    return np.linalg.norm(Y - ref) / np.linalg.norm(ref)


def test_smoothing_cuts_int8_error_on_outlier_channels():
    X = synth.activations(64, 512, 9, salient_frac=0.02, salient_mult=50.0)
    W = synth.weights(96, 512, 0.02, 9)
    plain = w8a8_error(X, W, oracle.INT8)
    s = oracle.smooth_scales(bits(X), bits(W), oracle.F16, 0.5)
    smooth = w8a8_error(X, W, oracle.INT8, s)
    assert smooth < 0.5 * plain, (smooth, plain)
    assert smooth < 0.05


def test_fp8_error_is_small_on_gaussian_data():
    X = synth.activations(32, 512, 10)
    W = synth.weights(64, 512, 0.02, 10)
    assert w8a8_error(X, W, oracle.E4M3) < 0.06
