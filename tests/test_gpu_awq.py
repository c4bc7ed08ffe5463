"""Parity of w4_awq_search (the AWQ alpha grid search) with the oracle,
through the C ABI.

Small layers: err[t] for every alpha within a relative 2e-3 of the oracle's
(the kernel path accumulates the layer in fp32 and the reference output in
fp32 where the oracle is exact; both round the layer output once to the
16-bit dtype), the same best index unless two errors tie within that
tolerance, best_scale bit-equal to the oracle's s at the best alpha, and the
optional quantized output bit-equal to the oracle's quantizer at that s.
Both GEMM paths run: Mc <= 32 (decode) and Mc > 32 (tcgen05).  The full-size
workload (512 x 4096 calibration rows, a 12288 x 4096 layer) is checked
against properties that hold at any size and a sampled estimate of err."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_pack_b200 as w4
from helpers import bits, odt

pytestmark = pytest.mark.gpu
DEV = "cuda"
RTOL = 2e-3


def run_case(Mc, N, K, sym, dtype, seed, alphas, quantize=True):
    W = synth.weights(N, K, 0.02, seed, outlier_frac=0.002, dtype=dtype)
    X = synth.activations(Mc, K, seed, salient_frac=0.02, dtype=dtype)
    err_o, s_o, best_o = oracle.awq_search(bits(W), bits(X), odt(W), 128, sym, alphas)
    out = w4.w4_awq_search(W.to(DEV), X.to(DEV), alphas, sym=sym, quantize=quantize)
    torch.cuda.synchronize()
    err = out[0].cpu().numpy()
    best = int(out[2].item())
    np.testing.assert_allclose(err, err_o, rtol=RTOL, err_msg=f"Mc={Mc} N={N} K={K}")
    if best != best_o:
        assert abs(err_o[best] - err_o[best_o]) <= RTOL * err_o[best_o], (best, best_o, err_o)
    np.testing.assert_array_equal(out[1].cpu().numpy(), s_o[best])
    if quantize:
        p, sc, z = oracle.quantize(bits(W), odt(W), 128, sym, s_o[best])
        assert np.array_equal(out[3][0].cpu().numpy(), p)
        assert np.array_equal(out[3][1].cpu().numpy(), sc)
        assert np.array_equal(out[3][2].cpu().numpy(), z)
    assert w4.w4_device_status() == w4.W4_OK
    return err, err_o


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("Mc,N,K", [(16, 96, 256), (5, 200, 384), (48, 130, 512),
                                    (200, 256, 1024)])
def test_search_parity(Mc, N, K, sym, dtype):
    run_case(Mc, N, K, sym, dtype, Mc + N + K, np.linspace(0.0, 1.0, 6))


def test_single_alpha_zero_is_plain_rtn():
    err, err_o = run_case(33, 64, 256, False, "f16", 3, [0.0], quantize=False)
    assert err[0] > 0


def test_ragged_and_tiny():
    run_case(1, 1, 128, True, "f16", 8, [0.0, 0.5, 1.0])
    run_case(32, 257, 128, False, "bf16", 9, [1.0, 0.25])
    run_case(33, 17, 640, False, "f16", 10, [0.3, 0.3, 0.7])


def test_repeated_calls_identical():
    Mc, N, K = 40, 300, 1024
    W = synth.weights(N, K, 0.02, 21).to(DEV)
    X = synth.activations(Mc, K, 21, salient_frac=0.02).to(DEV)
    ws = torch.empty(w4.w4_awq_search_workspace_bytes(Mc, K, N), dtype=torch.uint8, device=DEV)
    a = w4.w4_awq_search(W, X, np.linspace(0, 1, 5), workspace=ws)
    b = w4.w4_awq_search(W, X, np.linspace(0, 1, 5), workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_full_size_properties():
    c = synth.AWQ_SEARCH
    Mc, K, N = c["Mc"], c["K"], c["N"]
    W = synth.weights(N, K, c["std"], c["seed"], outlier_frac=c["w_outlier"], dtype=c["dtype"])
    X = synth.activations(Mc, K, c["seed"], salient_frac=c["x_salient"], dtype=c["dtype"])
    alphas = np.linspace(0.0, 1.0, c["n_alpha"]).astype(np.float32)
    err, s_best, best, (pk, sc, zp) = w4.w4_awq_search(W.to(DEV), X.to(DEV), alphas,
                                                       sym=c["sym"], quantize=True)
    torch.cuda.synchronize()
    err = err.cpu().numpy()
    best = int(best.item())
    assert np.isfinite(err).all() and (err > 0).all()
    assert best == int(np.argmin(err))
    # s at the best alpha: the column-mean ratio computed with numpy
    Xv = X.to(torch.float64).numpy()
    Wv = W.to(torch.float64).numpy()
    a = (np.abs(Xv).sum(0) / Mc).astype(np.float32).astype(np.float64)
    wm = (np.abs(Wv).sum(0) / N).astype(np.float32).astype(np.float64)
    want = np.power(a / wm, np.float64(alphas[best])).astype(np.float32)
    np.testing.assert_allclose(s_best.cpu().numpy(), want, rtol=2 ** -22)
    # the quantized output is the oracle's quantizer at that s
    p, s, z = oracle.quantize(bits(W), odt(W), 128, c["sym"], want)
    assert np.array_equal(pk.cpu().numpy(), p)
    # sampled estimate of err at the best alpha: 16384 (i, n) pairs through the oracle
    rng = np.random.default_rng(0)
    ii = rng.integers(0, Mc, 16384)
    nn = rng.integers(0, N, 16384)
    Xs = (Xv.astype(np.float32) / want).astype(np.float16)
    yq = oracle.linear_at(Xs.view(np.uint16), oracle.F16, p, s, z, 128, list(zip(ii, nn)))
    yq = yq.astype(np.float16).astype(np.float64)
    yref = np.einsum("ij,ij->i", Xv[ii], Wv[nn])
    est = ((yq - yref) ** 2).mean() * Mc * N
    assert abs(est - err[best]) <= 0.15 * err[best], (est, err[best])
    assert w4.w4_device_status() == w4.W4_OK
