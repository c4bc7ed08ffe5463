"""Property checks of the oracle on generated inputs (hypothesis): facts the
quantization formulas of "LLM quantization methods: principles and
implementation" §2.2 (symmetric / asymmetric INT4 and INT8) and §4.6 (FP8
E4M3) fix for every input, not only for the seeded cases of the other pin
files:
  * every INT4 code lies in its range and is a nearest level of w / s (+ zp),
    so |w - w^| <= s / 2 inside the representable range;
  * the group's extreme values land on the extreme codes (asymmetric: when
    the group straddles 0);
  * INT8 codes satisfy |v / scale - q| <= 1/2 and |q| <= 127, with the
    largest |v| on +-127;
  * an E4M3 code is the nearest E4M3 value of v / scale (no other code lies
    strictly closer), and the largest |v| maps to +-448.
"""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True, database=None,
                    suppress_health_check=[HealthCheck.too_slow])


def group_values(draw_scale, draw_vals):
    v = np.asarray(draw_vals, dtype=np.float64) * draw_scale
    return torch.from_numpy(v.reshape(1, -1)).to(torch.float16)


@st.composite
def fp16_group(draw, n=128):
    scale = draw(st.sampled_from([1e-4, 1e-2, 1.0, 30.0, 2000.0]))
    vals = draw(st.lists(st.floats(-1.0, 1.0, allow_nan=False, width=32), min_size=n, max_size=n))
    W = group_values(scale, vals)
    return W


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@SETTINGS
@given(W=fp16_group(), sym=st.booleans())
def test_int4_codes_are_in_range_and_nearest(W, sym):
    p, s, z = oracle.quantize(bits(W), oracle.F16, 128, sym)
    w = W.to(torch.float64).numpy()[0]
    u = np.array([oracle.code(p, 128, 0, k) for k in range(128)])
    s, z = float(s[0, 0]), float(z[0, 0])
    if sym:
        assert z == 8.0 and u.min() >= 1 and u.max() <= 15
    else:
        assert 0 <= z <= 15 and z == int(z) and u.min() >= 0 and u.max() <= 15
    if s == 0.0:
        assert (u == z).all()
        return
    wh = (u - z) * s
    lo, hi = (-7 * s, 7 * s) if sym else ((0 - z) * s, (15 - z) * s)
    inside = (w >= lo) & (w <= hi)
    # fp32 arithmetic of the quantizer: allow a few ulps of s beyond the exact half step
    assert (np.abs(w - wh)[inside] <= s * (0.5 + 1e-5)).all()
    # the extremes of the group sit on the extreme codes
    if sym:
        k = int(np.argmax(np.abs(w)))
        assert u[k] in (1, 15)
    elif w.min() < 0.0 < w.max():  # a group that straddles 0 uses the whole code range
        assert u[int(np.argmax(w))] >= 14 and u[int(np.argmin(w))] <= 1


@st.composite
def fp16_matrix(draw):
    rows = draw(st.integers(1, 4))
    scale = draw(st.sampled_from([1e-3, 1.0, 100.0]))
    vals = draw(st.lists(st.floats(-1.0, 1.0, allow_nan=False, width=32), min_size=rows * 32,
                         max_size=rows * 32))
    v = np.asarray(vals, dtype=np.float64).reshape(rows, 32) * scale
    return torch.from_numpy(v).to(torch.float16)


@SETTINGS
@given(A=fp16_matrix())
def test_int8_codes_round_to_nearest(A):
    q, sc = oracle.quant8(bits(A), oracle.F16, oracle.INT8)
    v = A.to(torch.float32).numpy()
    qi = q.view(np.int8).astype(np.float64)
    if sc == 0:
        assert not q.any()
        return
    assert np.abs(qi).max() == 127
    t = (v / np.float32(sc)).astype(np.float64)
    assert (np.abs(t - qi) <= 0.5).all() and (np.abs(qi) <= 127).all()


@SETTINGS
@given(A=fp16_matrix())
def test_e4m3_codes_are_nearest_values(A):
    q, sc = oracle.quant8(bits(A), oracle.F16, oracle.E4M3)
    if sc == 0:
        assert not q.any()
        return
    table = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    finite = ~np.isnan(table)
    t = (A.to(torch.float32).numpy() / np.float32(sc)).astype(np.float64).ravel()
    got = table[q.ravel()]
    assert np.abs(got).max() == 448.0
    best = np.min(np.abs(t[:, None] - table[None, finite]), axis=1)
    assert np.allclose(np.abs(t - got), best, rtol=0, atol=0)
