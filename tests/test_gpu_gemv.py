"""Parity of the small-M decode paths with the oracle's fp64 product, through
the C ABI: M = 1 with K % 512 == 0 (the CUDA-core GEMV) and every other
1 <= M <= 8 with K <= 4096 (the warp-level tensor-core GEMV); neither takes a
workspace.

The packed weights are the oracle's own quantization of seeded weights; the
tolerance is the W4A16 one of tests/helpers.py."""
import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(M, N, K, sym, dtype, seed, pass_zeros=True, x_salient=0.01, w_outlier=0.001, xscale=1.0,
        std=0.02):
    W = synth.weights(N, K, std, seed, outlier_frac=w_outlier, dtype=dtype)
    X = synth.activations(M, K, seed, salient_frac=x_salient, dtype=dtype)
    if xscale != 1.0:
        X = (X.float() * xscale).to(X.dtype)
        assert torch.isfinite(X).all(), "scaled activations must stay finite"
    packed, scales, zeros = oracle_quantize(W, 128, sym)
    z = zeros if (pass_zeros or not sym) else None
    pd = torch.from_numpy(packed).to(DEV)
    sd = torch.from_numpy(scales).to(DEV)
    zd = None if z is None else torch.from_numpy(z).to(DEV)
    assert w4.w4a16_workspace_bytes(M, K, N) == 0
    guard = 64
    buf = torch.full((M * N + 2 * guard,), 7.0, dtype=X.dtype, device=DEV)
    Y = buf[guard:guard + M * N].view(M, N)
    w4.w4a16_gemm(X.to(DEV), pd, sd, zd, out=Y)
    torch.cuda.synchronize()
    assert (buf[:guard] == 7.0).all() and (buf[-guard:] == 7.0).all(), "Y guard overwritten"
    check_y(Y, oracle_linear(X, packed, scales, z, K), f"M={M} N={N} K={K} sym={sym} {dtype}")
    return Y


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("K", [128, 384, 512, 1024, 1152, 2048, 2944, 3072, 4096])
def test_group_counts(K, sym, dtype):
    """Groups per warp from 0 to 4, odd group counts (4-byte scale copies)."""
    run(1, 333, K, sym, dtype, K + (7 if sym else 0) + (1 if dtype == "bf16" else 0))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_every_m(M, dtype):
    run(M, 1000, 4096, M % 2 == 0, dtype, 40 + M)


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("N", [1, 2, 7, 15, 16, 17, 147, 148, 149, 296, 443, 444, 445, 889, 1777, 2371,
                               4101])
def test_row_counts(N, M):
    """Rows per CTA from 1 to many (the M = 1 GEMV runs up to three CTAs per
    SM: N around 444 and its multiples gives CTAs of 1 to 5 rows and warps
    with none), partial batches of 4 rows (M = 1) and partial tiles of 16
    rows (M = 2)."""
    run(M, N, 4096, False, "f16", N + M)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_symmetric_without_zero_points(dtype):
    run(3, 500, 2048, True, dtype, 11, pass_zeros=False)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_large_activations(dtype):
    """Activations near the top of the 16-bit range and outlier channels."""
    run(2, 256, 4096, False, dtype, 12, x_salient=0.02, xscale=400.0)


def test_subnormal_activations():
    """fp16 activations mostly in the subnormal range (|x| < 2^-14): the
    products x * u * 2^-24 stay normal fp32 numbers, so nothing is flushed.
    Large weights keep the outputs in fp16's normal range."""
    run(1, 300, 1024, False, "f16", 13, x_salient=0.0, xscale=2.0 ** -16, std=4.0)


def test_repeated_calls_identical():
    N, K = 3000, 4096
    W = synth.weights(N, K, 0.02, 13)
    X = synth.activations(1, K, 13, salient_frac=0.01).to(DEV)
    packed, scales, zeros = oracle_quantize(W, 128, False)
    pd, sd, zd = (torch.from_numpy(a).to(DEV) for a in (packed, scales, zeros))
    a = w4.w4a16_gemm(X, pd, sd, zd)
    b = w4.w4a16_gemm(X, pd, sd, zd)
    assert torch.equal(a, b)
    assert w4.w4_device_status() == w4.W4_OK
