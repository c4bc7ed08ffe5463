"""Pins of the oracle's AWQ scale search to facts that do not come from the
oracle itself.

The search ("LLM quantization methods: principles and implementation",
§4.2 AWQ; "PTQ weight quantization: from GPTQ to AWQ", section "AWQ") picks,
over a grid of alpha, the per-input-channel factor s = (a / w)^alpha that
minimises || Q(W * s)(X / s) - W X ||.  The pins:
  * the 16-bit rounding it uses agrees with numpy / torch conversions;
  * s at alpha = 1 is the ratio of column means that numpy computes, alpha = 0
    gives s = 1, and a channel with no activation keeps s = 1;
  * at alpha = 0 the error is the plain RTN layer error computed with numpy
    from the (separately pinned) quantizer;
  * a weight matrix that lies on the INT4 grid after a power-of-two column
    scaling is reproduced exactly, so only the output rounding is left, the
    same at every alpha whose s is a power of two;
  * doubling X multiplies the error by exactly 4 at alpha in {0, 1};
  * on activations with salient channels a positive alpha beats plain RTN
    (the claim the method rests on).
A dropped fold, an inverted s, a mean over the wrong axis, a missing
division of X or a wrong rounding of the layer output fails one of them.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def vals(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def round_np(y: np.ndarray, dtype: int) -> np.ndarray:
    """Library rounding of exactly-fp32-representable values to the 16-bit dtype."""
    if dtype == oracle.F16:
        return y.astype(np.float16).astype(np.float64)
    return torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_round16_matches_library_conversion(dtype):
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 4, 2000),
                        [0.0, -0.0, 65504.0, 65519.0, 65520.0, -70000.0, 2.0 ** -25, 2.0 ** -26,
                         3 * 2.0 ** -26, 1e-30, 3.0e38, 3.4e38]]).astype(np.float32)
    got = np.array([oracle.round16(float(x), dtype) for x in v])
    want = round_np(v.astype(np.float64), dtype)
    np.testing.assert_array_equal(got, want)


def test_scale_formula_against_numpy_means():
    X = synth.activations(24, 384, 11, salient_frac=0.02)
    X[:, 5] = 0.0  # a channel the calibration data never excites
    W = synth.weights(40, 384, 0.02, 11)
    err, s, best = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, True, [0.0, 0.5, 1.0])
    a = (np.abs(vals(X)).sum(0) / 24).astype(np.float32)
    w = (np.abs(vals(W)).sum(0) / 40).astype(np.float32)
    ratio = a.astype(np.float64) / w.astype(np.float64)
    np.testing.assert_array_equal(s[0], np.ones(384, np.float32))
    want1 = ratio.astype(np.float32)
    want1[5] = 1.0
    np.testing.assert_array_equal(s[2], want1)
    want_half = np.sqrt(ratio).astype(np.float32)
    want_half[5] = 1.0
    np.testing.assert_allclose(s[1], want_half, rtol=2 ** -23)
    assert np.isfinite(err).all() and (err >= 0).all()


@pytest.mark.parametrize("sym", [True, False])
def test_alpha_zero_is_plain_rtn_error(sym):
    X = synth.activations(20, 256, 12, salient_frac=0.02)
    W = synth.weights(48, 256, 0.02, 12, outlier_frac=0.01)
    err, _, _ = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, sym, [0.0])
    p, sc, z = oracle.quantize(bits(W), oracle.F16, 128, sym)
    What = oracle.dequant(p, sc, None if sym else z, 256, 128)
    yq = round_np(vals(X) @ What.T, oracle.F16)
    yref = vals(X) @ vals(W).T
    want = ((yq - yref) ** 2).sum()
    np.testing.assert_allclose(err[0], want, rtol=1e-12)


def grid_case(sym: bool, dtype: str):
    """W = v / 8 on the INT4 grid (every row of every group holds the extreme
    code, so the group scale is exactly 1/8); the columns of X in group g are
    2^(e_g - 3) times a permutation of the same values v, so a_j / w_j = 2^e_g
    exactly."""
    v = np.array([7, -3, 1, -5, 2, 0, -6, 4] if sym else [7, -3, 1, -8, 2, 0, -6, 4], np.float64)
    N, Mc, K = 16, 16, 384
    e = np.repeat([-2, 0, 2], 128)
    n, j = np.meshgrid(np.arange(N), np.arange(K), indexing="ij")
    Wv = v[(n + j) % 8] / 8.0
    i, j = np.meshgrid(np.arange(Mc), np.arange(K), indexing="ij")
    Xv = v[(i + 3 * j) % 8] * 2.0 ** (e[None, :] - 3)
    dt = torch.float16 if dtype == "f16" else torch.bfloat16
    return torch.from_numpy(Wv).to(dt), torch.from_numpy(Xv).to(dt), Wv, Xv


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sym", [True, False])
def test_grid_weights_leave_only_output_rounding(sym, dtype):
    W, X, Wv, Xv = grid_case(sym, dtype)
    od = oracle.F16 if dtype == "f16" else oracle.BF16
    alphas = [0.0, 0.5, 1.0, 0.25]
    err, s, best = oracle.awq_search(bits(W), bits(X), od, 128, sym, alphas)
    # s_j = 2^(e_g * alpha)
    e = np.repeat([-2.0, 0.0, 2.0], 128)
    for t in range(3):
        np.testing.assert_array_equal(s[t], (2.0 ** (e * alphas[t])).astype(np.float32))
    y = Xv @ Wv.T
    rounding_only = ((round_np(y, od) - y) ** 2).sum()
    for t in range(3):
        assert err[t] == rounding_only, (t, err[t], rounding_only)
    # a factor of 2^(+-1/2) takes X / s off the bf16 grid: the error grows
    # (in fp16 the extra error stays below the output's rounding step here)
    if dtype == "bf16":
        assert err[3] > rounding_only
    assert best == 0 or err[best] == rounding_only


@pytest.mark.parametrize("sym", [True, False])
def test_doubling_activations_quadruples_error(sym):
    X = synth.activations(16, 256, 13, salient_frac=0.02)
    W = synth.weights(32, 256, 0.02, 13)
    alphas = [0.0, 1.0]
    e1, s1, _ = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, sym, alphas)
    e2, s2, _ = oracle.awq_search(bits(W), bits(X * 2), oracle.F16, 128, sym, alphas)
    np.testing.assert_array_equal(s2[1], s1[1] * 2)
    np.testing.assert_array_equal(e2, 4 * e1)


def test_salient_channels_prefer_positive_alpha():
    X = synth.activations(32, 512, 14, salient_frac=0.02)
    W = synth.weights(64, 512, 0.02, 14)
    alphas = np.linspace(0.0, 1.0, 11)
    err, _, best = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, False, alphas)
    assert best > 0 and err[best] < 0.8 * err[0]
    assert best == int(np.argmin(err))


def test_repeated_alpha_and_first_minimum():
    X = synth.activations(8, 256, 15, salient_frac=0.02)
    W = synth.weights(16, 256, 0.02, 15)
    err, s, best = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, True,
                                     [0.4, 0.0, 0.4, 0.4])
    assert err[0] == err[2] == err[3]
    np.testing.assert_array_equal(s[0], s[2])
    assert best == (0 if err[0] <= err[1] else 1)


def test_half_alpha_against_numpy_restatement():
    """Cross-check of the wiring (not a pin from the pages): the error at
    alpha = 0.5 assembled with numpy around the pinned quantizer."""
    X = synth.activations(12, 256, 16, salient_frac=0.02)
    W = synth.weights(24, 256, 0.02, 16)
    err, s, _ = oracle.awq_search(bits(W), bits(X), oracle.F16, 128, False, [0.5])
    a = (np.abs(vals(X)).sum(0) / 12).astype(np.float32).astype(np.float64)
    w = (np.abs(vals(W)).sum(0) / 24).astype(np.float32).astype(np.float64)
    sv = np.sqrt(a / w).astype(np.float32)
    p, sc, z = oracle.quantize(bits(W), oracle.F16, 128, False, sv)
    What = oracle.dequant(p, sc, z, 256, 128)
    Xs = (vals(X).astype(np.float32) / sv).astype(np.float16).astype(np.float64)
    yq = round_np(Xs @ What.T, oracle.F16)
    want = ((yq - vals(X) @ vals(W).T) ** 2).sum()
    np.testing.assert_allclose(err[0], want, rtol=1e-12)
