"""Parity of the decode path of w4a16_gemm (M <= 32, split-K tensor-core
GEMV) with the oracle's fp64 product, through the C ABI.

The packed weights fed to the CUDA kernel are the oracle's own quantization
of the seeded weights, so no oracle input comes from the CUDA path.
Tolerance: see tests/helpers.py (max error <= 1e-2 * max|Y_ref|, mean
relative error <= 1e-3 against Y_ref rounded once to the output dtype)."""
import numpy as np
import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_dev(packed, scales, zeros):
    z = None if zeros is None else torch.from_numpy(zeros).to(DEV)
    return torch.from_numpy(packed).to(DEV), torch.from_numpy(scales).to(DEV), z


def run_gemm(X, packed, scales, zeros, guard=64):
    """w4a16_gemm with guard elements around Y."""
    M = X.shape[0]
    N = packed.shape[0]
    buf = torch.full((M * N + 2 * guard,), 3.0, dtype=X.dtype, device=DEV)
    Y = buf[guard:guard + M * N].view(M, N)
    w4.w4a16_gemm(X, packed, scales, zeros, out=Y)
    torch.cuda.synchronize()
    assert (buf[:guard] == 3.0).all() and (buf[-guard:] == 3.0).all(), "Y guard overwritten"
    return Y


def case(M, N, K, sym, dtype, seed, std=0.02, w_outlier=0.0, x_salient=0.0, pass_zeros=True,
         rows=None):
    W = synth.weights(N, K, std, seed, outlier_frac=w_outlier, dtype=dtype)
    X = synth.activations(M, K, seed, salient_frac=x_salient, dtype=dtype)
    packed, scales, zeros = oracle_quantize(W, 128, sym)
    zarg = zeros if (pass_zeros or not sym) else None
    pd, sd, zd = to_dev(packed, scales, zarg)
    Y = run_gemm(X.to(DEV), pd, sd, zd)
    Yref = oracle_linear(X, packed, scales, zarg, K, 128, rows=rows)
    if rows is not None:
        Y = Y[:, torch.from_numpy(np.asarray(rows)).to(DEV)]
    return check_y(Y, Yref, f"M={M} N={N} K={K} sym={sym} {dtype}")


def test_tiny_workload_gemv():
    # 256 x 512 symmetric weights, X 1 x 512 fp16 ~ N(0, 1), seed 0
    c = synth.TINY
    case(1, c["N"], c["K"], True, "f16", c["seed"])


@pytest.mark.parametrize("N", synth.DECODE_M1["Ns"])
def test_decode_m1_full_size(N):
    c = synth.DECODE_M1
    case(1, N, c["K"], c["sym"], c["dtype"], c["seed"], c["std"], c["w_outlier"], c["x_salient"])


@pytest.mark.parametrize("M", synth.DECODE_SMALLM["Ms"])
def test_decode_small_m_full_size_sampled_rows(M):
    c = synth.DECODE_SMALLM
    rows = np.sort(np.random.default_rng(M).choice(c["N"], 384, replace=False))
    case(M, c["N"], c["K"], c["sym"], c["dtype"], c["seed"], c["std"], 0.0, c["x_salient"],
         rows=rows)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 13, 16, 17, 24, 25, 31, 32])
def test_ragged_m(dtype, M):
    case(M, 77, 384, False, dtype, 1000 + M, x_salient=0.02)


@pytest.mark.parametrize("N,K", [(1, 128), (15, 128), (17, 256), (200, 1152), (257, 4096),
                                 (1024, 4096), (4096, 256), (300, 16384)])
@pytest.mark.parametrize("M", [1, 7, 32])
def test_shapes(N, K, M):
    case(M, N, K, True, "f16", N * 7 + K + M, x_salient=0.01)


@pytest.mark.parametrize("M,N,K", [(1, 160000, 256), (2, 270000, 128), (5, 151553, 384)])
def test_whole_row_block_ranges(M, N, K):
    """Many row blocks per CTA (>= 8 per SM) or more row blocks than the
    workspace counter area holds: every CTA takes whole row blocks, no K is
    split across CTAs and no workspace is needed."""
    assert w4.w4a16_workspace_bytes(M, K, N) == 0
    case(M, N, K, False, "f16", N + K + M, x_salient=0.01)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_symmetric_without_zero_points(dtype):
    case(4, 96, 512, True, dtype, 5, pass_zeros=False)


def test_split_k_repeated_calls():
    """Shapes with few row tiles split K across CTAs (workspace path); the
    arrival counters must re-arm so that later calls stay correct."""
    M, N, K = 1, 512, 8192
    assert w4.w4a16_workspace_bytes(M, K, N) > 0
    W = synth.weights(N, K, 0.02, 9)
    packed, scales, zeros = oracle_quantize(W, 128, False)
    pd, sd, zd = to_dev(packed, scales, zeros)
    ws = w4.Workspace()
    outs = []
    for i in range(3):
        X = synth.activations(M, K, 20 + i, salient_frac=0.01)
        Y = w4.w4a16_gemm(X.to(DEV), pd, sd, zd, workspace=ws)
        torch.cuda.synchronize()
        check_y(Y, oracle_linear(X, packed, scales, zeros, K), f"call {i}")
        outs.append(Y.clone())
    X = synth.activations(M, K, 20, salient_frac=0.01)
    Y = w4.w4a16_gemm(X.to(DEV), pd, sd, zd, workspace=ws)
    assert torch.equal(Y, outs[0]), "split-K result is not deterministic"
    assert w4.w4_device_status() == 0


def test_deterministic():
    M, N, K = 3, 2048, 4096
    W = synth.weights(N, K, 0.02, 3)
    X = synth.activations(M, K, 3).to(DEV)
    packed, scales, zeros = oracle_quantize(W, 128, False)
    pd, sd, zd = to_dev(packed, scales, zeros)
    a = w4.w4a16_gemm(X, pd, sd, zd)
    b = w4.w4a16_gemm(X, pd, sd, zd)
    assert torch.equal(a, b)


def test_quantize_then_gemm_on_device():
    """The full path on the device: w4_quantize output feeds w4a16_gemm."""
    M, N, K = 2, 640, 2048
    W = synth.weights(N, K, 0.02, 31, outlier_frac=0.001)
    X = synth.activations(M, K, 31, salient_frac=0.01)
    packed, scales, zeros = w4.w4_quantize(W.to(DEV), 128, sym=False)
    Y = w4.w4a16_gemm(X.to(DEV), packed, scales, zeros)
    torch.cuda.synchronize()
    p, s, z = oracle_quantize(W, 128, False)
    assert np.array_equal(packed.cpu().numpy(), p)
    check_y(Y, oracle_linear(X, p, s, z, K), "device path")


def test_back_to_back_launches_overlap():
    """Layers launched one after another with no synchronization in between:
    with programmatic dependent launch a launch's CTAs start (and stream
    their weights) while the previous launch's CTAs finish on the same SMs,
    and wait for its tensor memory.  Every output must still match."""
    shapes = [(1, 1000, 1024), (1, 4096, 4096), (3, 2000, 2048), (1, 12288, 4096), (16, 700, 1024)]
    cases = []
    for i, (M, N, K) in enumerate(shapes):
        W = synth.weights(N, K, 0.02, 900 + i)
        X = synth.activations(M, K, 900 + i)
        packed, scales, zeros = oracle_quantize(W, 128, i % 2 == 0)
        pd, sd, zd = to_dev(packed, scales, zeros)
        cases.append((X, X.to(DEV), packed, scales, zeros, pd, sd, zd, K))
    outs = []
    for rep in range(3):
        outs.append([w4.w4a16_gemm(Xd, pd, sd, zd) for (_, Xd, _, _, _, pd, sd, zd, _) in cases])
    torch.cuda.synchronize()
    for rep in range(3):
        for (X, _, packed, scales, zeros, _, _, _, K), Y in zip(cases, outs[rep]):
            check_y(Y, oracle_linear(X, packed, scales, zeros, K, 128), f"back-to-back rep {rep}")
    assert w4.w4_device_status() == w4.W4_OK
