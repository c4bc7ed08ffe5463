"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or mathematics fix:
a worked example the pages print, special cases that reduce to a library
routine (numpy/torch rounding, float16 decoding, matmul), brute-force searches
over the 16 levels, and invariants of the method.  A plausible slip in the
oracle (a wrong divisor, a dropped zero point, a transposed nibble, rounding
half-up instead of half-to-even, a clamp on the wrong side) fails at least one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def f16(vals):
    return np.asarray(vals, dtype=np.float16)


def group_of(vals, group=128, fill=0.0):
    """One row holding `vals` first, padded with `fill` to a full group."""
    v = np.full(group, fill, dtype=np.float32)
    v[: len(vals)] = vals
    return f16(v).reshape(1, group)


# ---- number formats ----------------------------------------------------------------------

def test_f16_decoding_matches_numpy_for_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_bf16_decoding_matches_torch_for_every_pattern():
    bits = np.arange(1 << 16, dtype=np.int32).astype(np.int16)
    ref = torch.from_numpy(bits).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(b) & 0xFFFF) for b in bits])
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.isnan(got[~ok]).all()


# ---- the worked example the pages print --------------------------------------------------

def test_worked_example_int4():
    g = _read_golden("worked_example_int4.txt")
    val = {k: float(v[0]) for k, v in g.items()}
    tol = {k: float(v[1]) for k, v in g.items()}
    lo, hi, w = val["range_min"], val["range_max"], val["weight"]
    # 128 weights spread over [lo, hi], both ends and 0.7 included
    vals = np.linspace(lo, hi, 128)
    vals[1] = w
    W = group_of(vals)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=False)
    s, z = float(scales[0, 0]), float(zeros[0, 0])
    assert int(val["levels"]) == 16
    assert abs(s - val["scale"]) <= tol["scale"]
    u = oracle.code(packed, 128, 0, 1)
    assert u - z == val["signed_code"]
    deq = oracle.dequant(packed, scales, zeros, 128, 128)[0, 1]
    assert abs(deq - val["dequant"]) <= tol["dequant"]
    w16 = float(W[0, 1])
    assert abs((w16 - deq) - val["abs_error"]) <= tol["abs_error"]
    # exact bits of the reading: s = fl32(5/15), zero point rne(7.5) = 8
    assert np.float32(s) == np.float32(5.0) / np.float32(15.0)
    assert z == 8.0


# ---- special cases that reduce to a library rounding routine ---------------------------

TIES = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 3.5, -3.5, 4.5, 5.5, 6.5, -6.5, 0.25, 2.75, -3.25]


def test_symmetric_unit_scale_is_numpy_round_half_even():
    # amax = 7 exactly -> s = 1, so q must equal np.round (half to even)
    vals = np.array([7.0] + TIES + list(np.random.default_rng(1).uniform(-7, 7, 100)))
    W = group_of(vals)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=True)
    assert scales[0, 0] == 1.0 and zeros[0, 0] == 8.0
    w16 = W.astype(np.float64)[0]
    q_ref = np.clip(np.round(w16), -7, 7)
    q = np.array([oracle.code(packed, 128, 0, k) - 8 for k in range(128)])
    assert np.array_equal(q, q_ref)
    assert q[TIES.index(2.5) + 1] == 2 and q[TIES.index(-2.5) + 1] == -2
    assert q[TIES.index(3.5) + 1] == 4


def test_asymmetric_unit_scale_zero_point_zero():
    # min 0, max 15 -> s = 1, zp = 0, u = clamp(np.round(w), 0, 15)
    vals = np.array([0.0, 15.0] + [abs(t) for t in TIES] + [14.5, 7.5, 8.5])
    W = group_of(vals, fill=3.0)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=False)
    assert scales[0, 0] == 1.0 and zeros[0, 0] == 0.0
    w16 = W.astype(np.float64)[0]
    u = np.array([oracle.code(packed, 128, 0, k) for k in range(128)])
    assert np.array_equal(u, np.clip(np.round(w16), 0, 15))


def test_asymmetric_rounds_after_adding_the_zero_point():
    # min -1, max 14 -> s = 1, zp = 1; x = 2.5 -> round(2.5 + 1) = 4 (round-then-add gives 3)
    vals = np.array([-1.0, 14.0, 2.5, -0.5, 0.5, 4.5, 12.5])
    W = group_of(vals, fill=1.0)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=False)
    assert scales[0, 0] == 1.0 and zeros[0, 0] == 1.0
    u = [oracle.code(packed, 128, 0, k) for k in range(7)]
    w16 = W.astype(np.float64)[0, :7]
    assert u == list(np.clip(np.round(w16 + 1.0), 0, 15).astype(int))
    assert u[2] == 4


# ---- brute force over the levels on random groups -----------------------------------------

def _random_W(N, K, seed, std=0.02, outlier=0.01, dtype="f16"):
    return synth.weights(N, K, std, seed, outlier_frac=outlier, dtype=dtype)


def _codes(packed, K):
    N = packed.shape[0]
    return np.array([[oracle.code(packed, K, n, k) for k in range(K)] for n in range(N)])


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_symmetric_codes_are_nearest_level(dtype):
    K, N, g = 256, 24, 128
    Wt = _random_W(N, K, 11, dtype=dtype)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    dt = oracle.F16 if dtype == "f16" else oracle.BF16
    packed, scales, zeros = oracle.quantize(W, dt, g, sym=True)
    w = Wt.to(torch.float64).numpy()
    u = _codes(packed, K)
    assert (zeros == 8.0).all()
    for n in range(N):
        for gi in range(K // g):
            sl = slice(gi * g, (gi + 1) * g)
            amax = np.abs(w[n, sl]).max()
            s = float(scales[n, gi])
            # scale formula: s * 7 is amax up to the fp32 rounding of the division
            assert abs(s * 7 - amax) <= 7 * np.spacing(np.float32(s))
            q = u[n, sl] - 8
            assert q.min() >= -7 and q.max() <= 7
            # the amax element sits on the outermost level with its own sign
            i = np.argmax(np.abs(w[n, sl]))
            assert q[i] == (7 if w[n, sl][i] > 0 else -7)
            # brute force: no level is closer than the chosen one
            levels = np.arange(-7, 8) * s
            dist = np.abs(w[n, sl][:, None] - levels[None, :])
            best = dist.min(axis=1)
            chosen = np.abs(w[n, sl] - q * s)
            assert (chosen <= best + 1e-6 * s).all()
            assert (chosen <= s / 2 * (1 + 1e-6)).all()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_asymmetric_codes_are_nearest_level(dtype):
    K, N, g = 256, 24, 128
    Wt = _random_W(N, K, 12, dtype=dtype)
    Wt[3] += 0.05  # a few skewed rows
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    dt = oracle.F16 if dtype == "f16" else oracle.BF16
    packed, scales, zeros = oracle.quantize(W, dt, g, sym=False)
    w = Wt.to(torch.float64).numpy()
    u = _codes(packed, K)
    for n in range(N):
        for gi in range(K // g):
            sl = slice(gi * g, (gi + 1) * g)
            mn, mx = w[n, sl].min(), w[n, sl].max()
            s, z = float(scales[n, gi]), float(zeros[n, gi])
            assert abs(s * 15 - (mx - mn)) <= 15 * np.spacing(np.float32(s)) + np.spacing(np.float32(mx - mn))
            assert z == np.round(z) and 0 <= z <= 15
            if 0 < -mn / s < 15:
                assert abs(-mn / s - z) <= 0.5 + 1e-5
            # a group that straddles 0 has an unclamped zero point:
            # its min element codes to 0 and its max element to 14 or 15
            if mn <= 0 <= mx:
                assert u[n, sl][np.argmin(w[n, sl])] == 0
                assert u[n, sl][np.argmax(w[n, sl])] in (14, 15)
            else:
                assert z in (0.0, 15.0)
            levels = (np.arange(16) - z) * s
            dist = np.abs(w[n, sl][:, None] - levels[None, :])
            chosen = np.abs(w[n, sl] - (u[n, sl] - z) * s)
            assert (chosen <= dist.min(axis=1) + 1e-6 * s).all()


def test_degenerate_groups_dequantize_to_zero():
    W = np.zeros((2, 256), np.float16)
    W[1, :128] = 0.125  # constant group
    W[1, 128:] = -3.0
    ps, ss, zs = oracle.quantize(W[:1], oracle.F16, 128, sym=True)
    assert (ss == 0).all() and (zs == 8).all()
    assert all(oracle.code(ps, 256, 0, k) == 8 for k in range(256))
    pa, sa, za = oracle.quantize(W[1:], oracle.F16, 128, sym=False)
    assert (sa == 0).all() and (za == 0).all()
    assert all(oracle.code(pa, 256, 0, k) == 0 for k in range(256))
    assert not oracle.dequant(pa, sa, za, 256, 128).any()


def test_all_positive_group_clips_like_the_code_form():
    # zp = clamp(round(-min/s)) = 0 when min > 0: values below s/2 clip to 0
    vals = np.array([1.0, 16.0, 1.2, 8.0])
    W = group_of(vals, fill=4.0)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=False)
    assert scales[0, 0] == 1.0 and zeros[0, 0] == 0.0
    u = [oracle.code(packed, 128, 0, k) for k in range(4)]
    assert u == [1, 15, 1, 8]  # 16 clamps to 15


# ---- fold of a per-column factor ----------------------------------------------------------

@pytest.mark.parametrize("sym", [True, False])
def test_fold_by_unit_and_power_of_two_factors(sym):
    K, N = 256, 8
    Wt = _random_W(N, K, 21)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    base = oracle.quantize(W, oracle.F16, 128, sym)
    ones = oracle.quantize(W, oracle.F16, 128, sym, col_scale=np.ones(K, np.float32))
    for a, b in zip(base, ones):
        assert np.array_equal(a, b)
    # a power-of-two factor per group scales s exactly and leaves the codes alone
    f = np.repeat(np.array([4.0, 0.25], np.float32), 128)
    p2, s2, z2 = oracle.quantize(W, oracle.F16, 128, sym, col_scale=f)
    assert np.array_equal(p2, base[0]) and np.array_equal(z2, base[2])
    assert np.array_equal(s2, base[1] * np.array([4.0, 0.25], np.float32))


def test_fold_reconstruction_bound():
    # W-hat / s_k must approximate W within half a (folded) step of its group
    K, N = 256, 6
    Wt = _random_W(N, K, 22)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    cs = synth.awq_col_scale(synth.activations(64, K, 7, salient_frac=0.02)).numpy()
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, False, col_scale=cs)
    What = oracle.dequant(packed, scales, zeros, K, 128)
    w = Wt.to(torch.float64).numpy()
    err = np.abs(What / cs[None, :].astype(np.float64) - w)
    step = np.repeat(scales.astype(np.float64), 128, axis=1) / cs[None, :]
    assert (err <= step * (0.5 + 1e-5)).all()


# ---- packing -------------------------------------------------------------------------------

def test_pack_layout_golden():
    g = _read_golden("pack_layout.txt")
    codes = [int(c) for c in g["codes"]]
    expect = np.array([int(b, 16) for b in g["bytes"]], np.uint8)
    # an asymmetric group with min 0 and max 15 maps integer weights to themselves
    row = np.array(codes + [0.0] * 110 + [15.0, 0.0], np.float32)
    W = f16(row).reshape(1, 128)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, sym=False)
    assert scales[0, 0] == 1.0 and zeros[0, 0] == 0.0
    assert np.array_equal(packed[0, :8], expect)


def test_code_readback_inverts_packing():
    K, N = 256, 5
    Wt = _random_W(N, K, 31)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, False)
    # every byte's two nibbles must be codes that some (n, k) reads back, each exactly once
    u = _codes(packed, K)
    hist_bytes = np.bincount(np.concatenate([packed.ravel() & 15, packed.ravel() >> 4]), minlength=16)
    assert np.array_equal(hist_bytes, np.bincount(u.ravel(), minlength=16))


# ---- the linear layer ----------------------------------------------------------------------

@pytest.mark.parametrize("M,N", [(1, 16), (3, 7), (4, 16)])
def test_linear_matches_numpy_matmul(M, N):
    K = 256
    Wt = _random_W(N, K, 41 + M)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, False)
    What = oracle.dequant(packed, scales, zeros, K, 128)
    X = synth.activations(M, K, 5, salient_frac=0.02)
    Xb = X.view(torch.int16).numpy().view(np.uint16)
    Y = oracle.linear(Xb, oracle.F16, What)
    Yref = X.to(torch.float64).numpy() @ What.T
    assert np.allclose(Y, Yref, rtol=1e-12, atol=1e-12)
    # the same product straight from the packed weights
    pairs = [(m, n) for m in range(M) for n in range(N)]
    Yat = oracle.linear_at(Xb, oracle.F16, packed, scales, zeros, 128, pairs)
    assert np.array_equal(Yat, Y.ravel())
    # row subset
    Yr = oracle.linear(Xb, oracle.F16, What, rows=[M - 1])
    assert np.array_equal(Yr[0], Y[M - 1])


def test_dequant_symmetric_default_zero():
    K, N = 128, 4
    Wt = _random_W(N, K, 51)
    W = Wt.view(torch.int16).numpy().view(np.uint16)
    packed, scales, zeros = oracle.quantize(W, oracle.F16, 128, True)
    a = oracle.dequant(packed, scales, zeros, K, 128)
    b = oracle.dequant(packed, scales, None, K, 128)
    assert np.array_equal(a, b)


# ---- argument checks (the pages' `assert in_f % group_size == 0`) -----------------------------

def test_rejects_k_not_multiple_of_group():
    W = np.zeros((2, 192), np.float16)
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W, oracle.F16, 128, True)


def test_rejects_nonfinite_inputs():
    W = np.zeros((1, 128), np.float16)
    W[0, 5] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.quantize(W, oracle.F16, 128, True)
