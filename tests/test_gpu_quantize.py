"""Bit-exact parity of the CUDA quantizer (w4_quantize through the C ABI)
with the CPU oracle: packed bytes, fp32 scales and fp32 zero points."""
import numpy as np
import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_quantize(W, group, sym, col_scale=None, guard=64):
    """Runs the CUDA quantizer with guard bands around each output."""
    N, K = W.shape
    G = K // group
    pk = torch.full((N * K // 2 + 2 * guard,), 0xA5, dtype=torch.uint8, device=DEV)
    sc = torch.full((N * G + 2 * guard,), 7.25, dtype=torch.float32, device=DEV)
    zp = torch.full((N * G + 2 * guard,), -3.5, dtype=torch.float32, device=DEV)
    # keep the 16-byte alignment the ABI asks for: guard is a multiple of 16 elements
    w4.w4_quantize_into(W.to(DEV), pk[guard:guard + N * K // 2].view(N, K // 2),
                        sc[guard:guard + N * G].view(N, G), zp[guard:guard + N * G].view(N, G),
                        group=group, sym=sym,
                        col_scale=None if col_scale is None else col_scale.to(DEV))
    torch.cuda.synchronize()
    pk, sc, zp = pk.cpu(), sc.cpu(), zp.cpu()
    assert (pk[:guard] == 0xA5).all() and (pk[-guard:] == 0xA5).all(), "packed guard overwritten"
    assert (sc[:guard] == 7.25).all() and (sc[-guard:] == 7.25).all(), "scales guard overwritten"
    assert (zp[:guard] == -3.5).all() and (zp[-guard:] == -3.5).all(), "zeros guard overwritten"
    return (pk[guard:-guard].view(N, K // 2).numpy(), sc[guard:-guard].view(N, G).numpy(),
            zp[guard:-guard].view(N, G).numpy())


def assert_same(got, want, label=""):
    gp, gs, gz = got
    wp, ws, wz = want
    bad = np.argwhere(gp != wp)
    assert bad.size == 0, f"{label}: {len(bad)} packed bytes differ, first at {bad[:3].tolist()}"
    assert np.array_equal(gs.view(np.uint32), ws.view(np.uint32)), f"{label}: scales differ"
    assert np.array_equal(gz.view(np.uint32), wz.view(np.uint32)), f"{label}: zeros differ"


def test_tiny_workload_symmetric():
    # 256 x 512 fp16 ~ N(0, 0.02), seed 0, symmetric, group 128
    c = synth.TINY
    W = synth.weights(c["N"], c["K"], c["std"], c["seed"])
    assert_same(gpu_quantize(W, 128, True), oracle_quantize(W, 128, True), "tiny")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("group", [32, 64, 128, 256])
@pytest.mark.parametrize("fold", [False, True])
def test_ragged_shapes(dtype, sym, group, fold):
    # K = 1280 is not a multiple of the 1024-wide CTA strip; N = 37 is not a
    # multiple of the 32-row tile.
    N, K = 37, 1280
    W = synth.weights(N, K, 0.02, seed=100 + group, outlier_frac=0.01, dtype=dtype)
    cs = None
    if fold:
        cs = synth.awq_col_scale(synth.activations(64, K, 7, salient_frac=0.02))
    assert_same(gpu_quantize(W, group, sym, cs), oracle_quantize(W, group, sym, cs),
                f"{dtype} sym={sym} g={group} fold={fold}")


@pytest.mark.parametrize("N,K", [(1, 128), (1, 4096), (33, 256), (513, 3072), (64, 11008)])
def test_more_shapes(N, K):
    W = synth.weights(N, K, 0.02, seed=N + K, outlier_frac=0.001)
    for sym in (True, False):
        assert_same(gpu_quantize(W, 128, sym), oracle_quantize(W, 128, sym), f"{N}x{K} sym={sym}")


def edge_matrix(dtype=torch.float16):
    """Rows that exercise every special case of the definition."""
    g = 128
    rows = []
    f = torch.finfo(dtype)
    rows.append(torch.zeros(g))                                     # all-zero group
    rows.append(torch.full((g,), 0.125))                            # constant positive
    rows.append(torch.full((g,), -3.0))                             # constant negative
    rows.append(torch.linspace(0.5, 4.0, g))                        # all positive
    rows.append(torch.linspace(-9.0, -1.0, g))                      # all negative
    # dtype extremes, kept inside the precondition that max - min is finite in fp32
    top = f.max if dtype == torch.float16 else f.max / 4
    rows.append(torch.tensor([top, -top] + [1.0] * (g - 2)))
    sub = f.tiny * torch.arange(-64, 64).float() / 64               # subnormals
    rows.append(sub)
    rows.append(torch.tensor([7.0] + [k + 0.5 for k in range(-7, 7)] * 9 + [0.0] * (g - 127)))  # ties, s=1
    rows.append(torch.tensor([-1.0, 14.0] + [k + 0.5 for k in range(-1, 14)] * 8 + [0.0] * (g - 122)))  # asym ties, s=1, zp=1
    rows.append(torch.linspace(-2.5, 2.5, g))                       # the worked example's range
    big = torch.zeros(g)
    big[0] = 1000.0
    big[1:] = torch.linspace(-1e-3, 1e-3, g - 1)                     # one dominant outlier
    rows.append(big)
    return torch.stack(rows).to(dtype)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("sym", [True, False])
def test_edge_matrix(dtype, sym):
    W = edge_matrix(dtype)
    W = torch.cat([W, W.flip(1)], dim=1)  # K = 256, two groups per row
    assert_same(gpu_quantize(W, 128, sym), oracle_quantize(W, 128, sym), f"edge {dtype} sym={sym}")


def _nudge(v, d):
    """Move each fp32 v by d ulps (d in -3..3)."""
    v = v.copy()
    for step in range(3):
        up = d > step
        dn = d < -step
        v[up] = np.nextafter(v[up], np.float32(np.inf))
        v[dn] = np.nextafter(v[dn], np.float32(-np.inf))
    return v


@pytest.mark.parametrize("sym", [True, False])
def test_values_next_to_rounding_boundaries(sym):
    """Folded weights placed within 3 ulps of the rounding boundaries
    (k + 1/2 steps), where a reciprocal product and the correctly rounded
    division can disagree.  The fp32 values enter through the column factor:
    W holds +-1, +-2, 1/2, so w * col_scale[k] is exact."""
    rng = np.random.default_rng(7)
    G = 64
    K = 128 * G
    cs = np.zeros(K, np.float32)
    for gi in range(G):
        lo, hi = (-1.0, 1.0) if sym else sorted(rng.uniform(-2.0, 2.0, 2))
        amax = np.float32(rng.uniform(0.05, 3.0))
        if sym:
            mx, mn = amax, np.float32(-0.9) * amax
            s = amax / np.float32(7.0)
            zp = np.float32(0.0)
            k = rng.integers(-7, 7, 126).astype(np.float32)
        else:
            mx, mn = np.float32(hi), np.float32(lo)
            s = (mx - mn) / np.float32(15.0)
            zp = np.float32(np.clip(np.round(-mn / s), 0, 15))
            k = rng.integers(0, 15, 126).astype(np.float32) - zp
        v = (k + np.float32(0.5)) * s
        v = _nudge(v.astype(np.float32), rng.integers(-3, 4, 126))
        v = np.clip(v, mn, mx)
        cs[gi * 128:(gi + 1) * 128] = np.concatenate([[mx, mn], v])
    W = torch.tensor([[1.0], [-1.0], [2.0], [0.5], [-2.0]], dtype=torch.float16).repeat(1, K)
    col = torch.from_numpy(cs)
    assert_same(gpu_quantize(W, 128, sym, col), oracle_quantize(W, 128, sym, col), "near-boundary")


def _fp16_magnitudes():
    """All positive finite fp16 values, ascending (31743 of them)."""
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    allv = allv[np.isfinite(allv)]
    return np.unique(np.abs(allv[allv != 0]))


def _sweep_chunk(P, i0, i1):
    """Groups [amax, x_1 .. x_127] for amax = P[i], i0 <= i < i1, whose x run
    over every fp16 value with |x| <= amax: 0, +-P[0..i]; padded with zeros."""
    blocks = []
    for i in range(i0, i1):
        xs = np.concatenate([[np.float16(0)], P[:i + 1], -P[:i + 1]])
        ng = (xs.size + 126) // 127
        xs = np.concatenate([xs, np.zeros(ng * 127 - xs.size, np.float16)]).reshape(ng, 127)
        blocks.append(np.concatenate([np.full((ng, 1), P[i], np.float16), xs], axis=1))
    W = np.concatenate(blocks)
    pad = (-W.shape[0]) % 8  # 8 groups per row
    W = np.concatenate([W, np.zeros((pad, 128), np.float16)]).reshape(-1, 1024)
    return torch.from_numpy(W)


def test_symmetric_code_map_over_all_fp16_values():
    """The symmetric scale -> code map exhaustively: every finite fp16 x
    against every positive finite fp16 amax (about 10^9 pairs, in chunks).
    Each group is [amax, x_1..x_127] with |x_i| <= amax, so the code of every
    x is decided by the scale fl(amax / 7) alone; codes, packed bytes and the
    scales are compared bit for bit with the oracle."""
    P = _fp16_magnitudes()
    assert P.size == 31743
    # chunk boundaries holding about 2^26 weights each (the work of amax i
    # grows like i)
    cum = np.cumsum(2 * np.arange(P.size) + 3)
    bounds = [0] + list(np.searchsorted(cum, np.arange(1, 64) * (cum[-1] / 64))) + [P.size]
    bounds = sorted(set(int(x) for x in bounds))
    pairs = 0
    for i0, i1 in zip(bounds[:-1], bounds[1:]):
        W = _sweep_chunk(P, i0, i1)
        pairs += int(cum[i1 - 1] - (cum[i0 - 1] if i0 else 0))
        assert_same(gpu_quantize(W, 128, True), oracle_quantize(W, 128, True),
                    f"fp16 sweep amax {P[i0]}..{P[i1 - 1]}")
    assert pairs > 10 ** 9


def test_7b_layer_full_size_sampled_rows():
    """One layer of the 7B stack at full size, AWQ factor folded, asymmetric.
    Rows are independent, so the oracle quantizes a seeded sample of rows."""
    c = synth.STACK_7B
    Xcal = synth.activations(c["calib_M"], 4096, c["seed"], salient_frac=c["x_salient"],
                             tensor_id=2)
    cs = synth.awq_col_scale(Xcal)
    rng = np.random.default_rng(0)
    for li, (name, out_f, in_f) in enumerate(c["shapes"]):
        W = synth.weights(out_f, in_f, c["std"], c["seed"], outlier_frac=c["w_outlier"],
                          device=DEV, tensor_id=16 + li)
        col = cs.to(DEV) if in_f == 4096 else None
        packed, scales, zeros = w4.w4_quantize(W, 128, sym=False, col_scale=col)
        torch.cuda.synchronize()
        rows = np.sort(rng.choice(out_f, 96, replace=False))
        Ws = W[torch.from_numpy(rows).to(DEV)].cpu()
        want = oracle_quantize(Ws, 128, False, None if col is None else cs)
        got = (packed.cpu().numpy()[rows], scales.cpu().numpy()[rows], zeros.cpu().numpy()[rows])
        assert_same(got, want, name)


def test_repeated_calls_identical():
    W = synth.weights(300, 2048, 0.02, seed=77, outlier_frac=0.001)
    a = gpu_quantize(W, 128, False)
    b = gpu_quantize(W, 128, False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
