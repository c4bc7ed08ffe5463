"""Pins of the oracle's GPTQ ("LLM quantization methods: principles and
implementation" §4.1; "PTQ weight quantization: from GPTQ to AWQ", section
"GPTQ") to facts that do not come from the oracle itself:
  * H = 2 X^T X against numpy's matmul, and the damped inverse factor U
    satisfies U^T U (H + lambda I) = I;
  * with a diagonal Hessian no error crosses columns, so GPTQ is exactly the
    RTN quantizer (pinned elsewhere);
  * the oracle's Cholesky-row, lazy-batched fp32 loop agrees with the pages'
    own update written out in numpy fp64 -- delta_j = (w_j - q_j) / [H_F^-1]_jj,
    W[:, F] -= delta_j [H_F^-1]_{j,F}, then column j removed from H_F^-1 --
    on the codes and the layer error;
  * on the calibration data GPTQ's layer error is far below RTN's (the method's
    claim), for symmetric and asymmetric storage.
A wrong update sign, a missing division by the diagonal, an update of the
wrong columns or group parameters taken from the original weights fails one.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import synth


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def vals(t):
    return t.to(torch.float64).numpy()


def test_hessian_and_factor():
    X = synth.activations(48, 128, 2, salient_frac=0.02)
    H = oracle.gptq_hessian(bits(X), oracle.F16)
    np.testing.assert_array_equal(H, 2.0 * vals(X).T @ vals(X))
    U = oracle.gptq_inverse_factor(H, 0.01)
    assert np.allclose(np.tril(U, -1), 0.0)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(128)
    np.testing.assert_allclose(U.T @ U @ Hd, np.eye(128), atol=1e-8)


@pytest.mark.parametrize("K,Mc,seed", [(128, 48, 2), (256, 512, 3), (384, 200, 4)])
def test_reversed_cholesky_gives_the_same_factor(K, Mc, seed):
    """The route the library's device code takes to U, checked in fp64 with
    numpy's and scipy's own routines: with P the index reversal and L the lower Cholesky
    factor of P (H + lambda I) P, P L^-1 P is upper triangular with a positive
    diagonal and (P L^-1 P)^T (P L^-1 P) = (H + lambda I)^-1, so by the
    uniqueness of the Cholesky factor it is the oracle's U."""
    X = synth.activations(Mc, K, seed, salient_frac=0.02)
    H = oracle.gptq_hessian(bits(X), oracle.F16)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(K)
    P = np.eye(K)[::-1]
    L = np.linalg.cholesky(P @ Hd @ P)
    Ur = P @ scipy.linalg.solve_triangular(L, np.eye(K), lower=True) @ P
    assert np.allclose(np.tril(Ur, -1), 0.0, atol=0.0)
    assert (np.diag(Ur) > 0).all()
    U = oracle.gptq_inverse_factor(H, 0.01)
    np.testing.assert_allclose(Ur, U, rtol=0, atol=1e-9 * np.abs(U).max())


@pytest.mark.parametrize("sym", [True, False])
def test_diagonal_hessian_is_rtn(sym):
    K = 256
    X = torch.eye(K, dtype=torch.float16) * 3  # orthogonal columns: H diagonal
    W = synth.weights(24, K, 0.02, 3, outlier_frac=0.01)
    p, s, z, U = oracle.gptq(bits(W), bits(X), oracle.F16, 128, sym)
    assert not np.triu(U, 1).any()
    pr, sr, zr = oracle.quantize(bits(W), oracle.F16, 128, sym)
    np.testing.assert_array_equal(p, pr)
    np.testing.assert_array_equal(s, sr)


def obs_reference(Wv, H, group, sym, percdamp=0.01):
    """The pages' update, fp64, no batching: for j in order, quantize w_j with
    its group's parameters (taken from the current weights when the group
    starts), delta = (w_j - q_j) / Hinv_jj, update the remaining columns with
    Hinv row j, then remove column j from Hinv."""
    N, K = Wv.shape
    Hd = H + percdamp * np.mean(np.diag(H)) * np.eye(K)
    Hinv = np.linalg.inv(Hd)
    W = Wv.copy()
    codes = np.zeros((N, K), np.int64)
    scales = np.zeros((N, K // group))
    deq = np.zeros((N, K))
    for j in range(K):
        if j % group == 0:
            blk = W[:, j:j + group].astype(np.float32)
            if sym:
                s = np.abs(blk).max(1) / np.float32(7)
                z = np.full(N, 8.0, np.float32)
            else:
                mn, mx = blk.min(1), blk.max(1)
                s = (mx - mn) / np.float32(15)
                with np.errstate(divide="ignore", invalid="ignore"):
                    z = np.where(s == 0, 0, np.clip(np.round(-mn / s), 0, 15)).astype(np.float32)
            scales[:, j // group] = s
        wj = W[:, j].astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            if sym:
                u = np.where(s == 0, 8, np.clip(np.round(wj / s), -7, 7) + 8)
            else:
                u = np.where(s == 0, 0, np.clip(np.round(wj / s + z), 0, 15))
        codes[:, j] = u
        q = (u - z.astype(np.float64)) * s.astype(np.float64)
        deq[:, j] = q
        delta = (W[:, j] - q) / Hinv[j, j]
        W[:, j + 1:] -= np.outer(delta, Hinv[j, j + 1:])
        Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / Hinv[j, j]
    return codes, scales, deq


def unpack(p, K):
    N = p.shape[0]
    return np.array([[oracle.code(p, K, n, k) for k in range(K)] for n in range(N)])


@pytest.mark.parametrize("sym", [True, False])
def test_agrees_with_the_pages_update(sym):
    K, N = 256, 12
    X = synth.activations(96, K, 4, salient_frac=0.02)
    W = synth.weights(N, K, 0.02, 4, outlier_frac=0.01)
    H = oracle.gptq_hessian(bits(X), oracle.F16)
    p, s, z, U = oracle.gptq(bits(W), bits(X), oracle.F16, 128, sym)
    codes_ref, scales_ref, deq_ref = obs_reference(vals(W), H, 128, sym)
    codes = unpack(p, K)
    assert (codes == codes_ref).mean() >= 0.995, (codes != codes_ref).sum()
    np.testing.assert_allclose(s, scales_ref, rtol=1e-4)
    # the layer error on the calibration data agrees too
    Xv = vals(X)
    Wq = oracle.dequant(p, s, None if sym else z, K, 128)
    e_oracle = np.linalg.norm((Wq - vals(W)) @ Xv.T)
    e_ref = np.linalg.norm((deq_ref - vals(W)) @ Xv.T)
    assert abs(e_oracle - e_ref) <= 0.02 * e_ref


@pytest.mark.parametrize("sym", [True, False])
def test_beats_rtn_on_calibration_data(sym):
    K, N = 512, 40
    X = synth.activations(256, K, 5, salient_frac=0.02)
    W = synth.weights(N, K, 0.02, 5, outlier_frac=0.001)
    p, s, z, U = oracle.gptq(bits(W), bits(X), oracle.F16, 128, sym)
    pr, sr, zr = oracle.quantize(bits(W), oracle.F16, 128, sym)
    Xv, Wv = vals(X), vals(W)
    err = lambda p, s, z: np.linalg.norm((oracle.dequant(p, s, None if sym else z, K, 128) - Wv) @ Xv.T)
    assert err(p, s, z) < 0.6 * err(pr, sr, zr)


def exact_case(N, K, sym, seed, group=128):
    """Weights and a factor U on which every fp32 and fp64 operation of the
    GPTQ update is exact, so the oracle's fp32 loop and the pages' fp64
    recursion must give the same codes and scales bit for bit.

    Per group: two anchor columns hold the group's extremes (-0.5 and 7/16,
    or +-7/16 symmetric), so its scale is 1/16 and its zero point 8; every
    other weight is a multiple of 2^-10 well inside that range.  Columns are
    sources (their errors are pushed onward) or sinks (they receive errors and
    push none): U is upper triangular with diagonal 1/2, 1 or 2 and a few
    off-diagonal entries +-1/8, +-1/16 from sources to later sinks, in the
    same and in later 128-column blocks.  Errors are then multiples of 2^-11,
    updates of 2^-15, and no sink leaves the anchors' range."""
    rng = np.random.default_rng(seed)
    W = np.round(rng.uniform(-0.35, 0.3, (N, K)) * 1024) / 1024
    role = rng.integers(0, 2, K)  # 1 = source
    for g in range(K // group):
        a = g * group + rng.choice(group, 2, replace=False)
        W[:, a[0]] = -7 / 16 if sym else -0.5
        W[:, a[1]] = 7 / 16
        role[a] = 2  # anchors: neither updated nor pushing (their error is 0 anyway)
    U = np.diag(rng.choice([0.5, 1.0, 2.0], K))
    for k in range(K):
        if role[k] != 0:
            continue
        srcs = [j for j in range(k) if role[j] == 1]
        for j in rng.choice(srcs, min(3, len(srcs)), replace=False) if srcs else []:
            U[j, k] = rng.choice([0.125, -0.125, 0.0625, -0.0625])
    return W, U


@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("N,K,seed", [(6, 256, 1), (10, 384, 2), (4, 512, 3), (16, 256, 4)])
def test_exact_against_the_pages_update(N, K, seed, sym):
    Wv, U = exact_case(N, K, sym, seed)
    W16 = torch.from_numpy(Wv).to(torch.float16)
    assert np.array_equal(vals(W16), Wv)  # the weights are exact in fp16
    p, s, z = oracle.gptq_quantize(bits(W16), oracle.F16, U.astype(np.float32), 128, sym)
    # the pages' recursion with H^-1 = U^T U given directly (no damping)
    codes_ref, scales_ref = pages_update(Wv, U.T @ U, 128, sym)
    np.testing.assert_array_equal(unpack(p, K), codes_ref)
    np.testing.assert_array_equal(s.astype(np.float64), scales_ref)
    assert np.all(s == np.float32(1 / 16))
    # some errors really crossed columns and blocks (the case is not trivial)
    pr, sr, zr = oracle.quantize(bits(W16), oracle.F16, 128, sym)
    assert not np.array_equal(p, pr)


def pages_update(Wv, Hinv, group, sym, mistake=None):
    """The pages' recursion (as obs_reference) with H^-1 given directly, fp64.
    `mistake` plants one error for the sensitivity check: "sign" (errors
    added instead of subtracted), "nodiv" (no division by [H_F^-1]_jj),
    "stale" (column j never removed from H_F^-1)."""
    N, K = Wv.shape
    Hinv = Hinv.copy()
    W = Wv.copy()
    codes = np.zeros((N, K), np.int64)
    scales = np.zeros((N, K // group))
    for j in range(K):
        if j % group == 0:
            blk = W[:, j:j + group].astype(np.float32)
            if sym:
                s = np.abs(blk).max(1) / np.float32(7)
                z = np.full(N, 8.0, np.float32)
            else:
                mn, mx = blk.min(1), blk.max(1)
                s = (mx - mn) / np.float32(15)
                z = np.clip(np.round(-mn / s), 0, 15).astype(np.float32)
            scales[:, j // group] = s
        wj = W[:, j].astype(np.float32)
        u = np.clip(np.round(wj / s), -7, 7) + 8 if sym else np.clip(np.round(wj / s + z), 0, 15)
        codes[:, j] = u
        q = (u - z.astype(np.float64)) * s.astype(np.float64)
        delta = (W[:, j] - q) / (1.0 if mistake == "nodiv" else Hinv[j, j])
        upd = np.outer(delta, Hinv[j, j + 1:])
        W[:, j + 1:] += upd if mistake == "sign" else -upd
        if mistake != "stale":
            Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / Hinv[j, j]
    return codes, scales


@pytest.mark.parametrize("mistake", ["sign", "nodiv", "stale"])
def test_exact_case_catches_planted_mistakes(mistake):
    """The exact construction is sensitive to the update it checks: each
    planted mistake in the pages' recursion changes the codes."""
    Wv, U = exact_case(8, 256, False, 5)
    W16 = torch.from_numpy(Wv).to(torch.float16)
    p, s, z = oracle.gptq_quantize(bits(W16), oracle.F16, U.astype(np.float32), 128, False)
    good, _ = pages_update(Wv, U.T @ U, 128, False)
    bad, _ = pages_update(Wv, U.T @ U, 128, False, mistake)
    np.testing.assert_array_equal(unpack(p, 256), good)
    assert not np.array_equal(good, bad)
