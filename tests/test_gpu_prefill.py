"""Parity of the prefill path of w4a16_gemm (M > 32: tcgen05 tensor cores,
TMEM accumulators, TMA-staged X) with the oracle's fp64 product, through
the C ABI.  Weights are the oracle's own quantization of the seeded weights.
Tolerance: see tests/helpers.py."""
import numpy as np
import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(M, N, K, sym, dtype, seed, pass_zeros=True, rows=None, std=0.02, x_salient=0.01):
    W = synth.weights(N, K, std, seed, dtype=dtype)
    X = synth.activations(M, K, seed, salient_frac=x_salient, dtype=dtype)
    packed, scales, zeros = oracle_quantize(W, 128, sym)
    zarg = zeros if (pass_zeros or not sym) else None
    guard = 64
    buf = torch.full((M * N + 2 * guard,), 5.0, dtype=X.dtype, device=DEV)
    Y = buf[guard:guard + M * N].view(M, N)
    w4.w4a16_gemm(X.to(DEV), torch.from_numpy(packed).to(DEV), torch.from_numpy(scales).to(DEV),
                  None if zarg is None else torch.from_numpy(zarg).to(DEV), out=Y)
    torch.cuda.synchronize()
    assert (buf[:guard] == 5.0).all() and (buf[-guard:] == 5.0).all(), "Y guard overwritten"
    assert w4.w4_device_status() == w4.W4_OK
    Yref = oracle_linear(X, packed, scales, zarg, K, 128, rows=rows)
    if rows is not None:
        Y = Y[:, torch.from_numpy(np.asarray(rows)).to(DEV)]
    return check_y(Y, Yref, f"M={M} N={N} K={K} sym={sym} {dtype}")


def test_single_tile():
    run(256, 128, 256, False, "bf16", 1)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("sym", [False, True])
def test_multi_tile(dtype, sym):
    run(512, 384, 1024, sym, dtype, 2)


@pytest.mark.parametrize("M,N,K", [(33, 1, 128), (40, 100, 128), (255, 129, 256), (257, 128, 384),
                                   (600, 300, 1152), (1000, 777, 512), (64, 4096, 4096)])
def test_ragged(M, N, K):
    run(M, N, K, False, "bf16", M + N + K)


def test_symmetric_without_zero_points():
    run(300, 200, 512, True, "bf16", 8, pass_zeros=False)


def test_prefill_workload_full_size_sampled_rows():
    # M = 2048, K = 4096, N = 11008, bf16, asymmetric, X with 1% channels x20
    c = synth.PREFILL
    rows = np.sort(np.random.default_rng(4).choice(c["N"], 192, replace=False))
    run(c["M"], c["N"], c["K"], c["sym"], c["dtype"], c["seed"], rows=rows, std=c["std"],
        x_salient=c["x_salient"])


def test_repeated_calls_identical():
    M, N, K = 512, 512, 2048
    W = synth.weights(N, K, 0.02, 5, dtype="bf16")
    X = synth.activations(M, K, 5, dtype="bf16").to(DEV)
    p, s, z = w4.w4_quantize(W.to(DEV), 128, sym=False)
    a = w4.w4a16_gemm(X, p, s, z)
    b = w4.w4a16_gemm(X, p, s, z)
    assert torch.equal(a, b)
