"""Parity of GPTQ on the GPU (w4_gptq_quantize, w4_gptq) with the oracle,
through the C ABI.

The column loop is a fixed function of W and the factor U (every update an
fp32 fma in a defined order, IEEE division), so given the same fp32 U the
GPU's codes, scales and zero points are bit-equal to the oracle's:
  * w4_gptq_quantize is run on the oracle's own U (fp64 factor rounded to fp32);
  * the whole w4_gptq computes H and U on the device in fp32; its U is
    copied back, checked within 2e-3 (relative to max |U|) of the oracle's
    fp64 factor, and the oracle's column loop run on that very U must give
    the GPU's codes, scales and zero points bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_pack_b200 as w4
from helpers import bits, odt

pytestmark = pytest.mark.gpu
DEV = "cuda"


def layer(N, K, Mc, dtype, seed):
    W = synth.weights(N, K, 0.02, seed, outlier_frac=0.002, dtype=dtype)
    X = synth.activations(Mc, K, seed, salient_frac=0.02, dtype=dtype)
    return W, X


def oracle_u32(X, percdamp=0.01):
    return oracle.gptq_inverse_factor(oracle.gptq_hessian(bits(X), odt(X)), percdamp).astype(np.float32)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K,Mc", [(1, 128, 64), (8, 256, 512), (33, 384, 200), (200, 1024, 256),
                                    (1000, 512, 1024)])
def test_column_loop_bit_exact(N, K, Mc, sym, dtype):
    W, X = layer(N, K, Mc, dtype, N + K + Mc)
    U = oracle_u32(X)
    p, s, z = w4.w4_gptq_quantize(W.to(DEV), torch.from_numpy(U).to(DEV), sym=sym)
    torch.cuda.synchronize()
    po, so, zo = oracle.gptq_quantize(bits(W), odt(W), U, 128, sym)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(z.cpu().numpy(), zo)
    assert np.array_equal(p.cpu().numpy(), po)
    assert w4.w4_device_status() == w4.W4_OK


def calib_error(packed, scales, zeros, W, X, K, sym):
    Wh = oracle.dequant(packed, scales, None if sym else zeros, K, 128)
    return np.linalg.norm((Wh - W.to(torch.float64).numpy()) @ X.to(torch.float64).numpy().T)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("N,K,Mc", [(64, 256, 512), (300, 512, 1024), (96, 512, 256),
                                    (40, 384, 256), (24, 640, 300)])
def test_whole_pipeline(N, K, Mc, sym):
    """K = 384 and 640 (6 and 10 diagonal blocks of 64) run the triangular
    inverse's partial last pair and its unpaired last block."""
    W, X = layer(N, K, Mc, "f16", 7 + N + K)
    p, s, z, U = w4.w4_gptq(W.to(DEV), X.to(DEV), sym=sym, return_u=True)
    torch.cuda.synchronize()
    Uo = oracle.gptq_inverse_factor(oracle.gptq_hessian(bits(X), odt(X)), 0.01)
    Ug32 = U.cpu().numpy()
    assert not np.tril(Ug32, -1).any()
    assert np.abs(Ug32.astype(np.float64) - Uo).max() <= 2e-3 * np.abs(Uo).max()
    # the oracle's column loop on the GPU's own factor: bit-equal
    po, so, zo = oracle.gptq_quantize(bits(W), odt(W), Ug32, 128, sym)
    pg, sg, zg = p.cpu().numpy(), s.cpu().numpy(), z.cpu().numpy()
    assert np.array_equal(sg, so)
    assert np.array_equal(zg, zo)
    assert np.array_equal(pg, po)
    # and the method's claim: below RTN's calibration error
    e_gpu = calib_error(pg, sg, zg, W, X, K, sym)
    pr, sr, zr = oracle.quantize(bits(W), odt(W), 128, sym)
    assert e_gpu < calib_error(pr, sr, zr, W, X, K, sym)


def test_not_positive_definite_is_reported():
    W = synth.weights(16, 256, 0.02, 3).to(DEV)
    X = torch.zeros(64, 256, dtype=torch.float16, device=DEV)
    with pytest.raises(w4.W4Error, match="positive definite"):
        w4.w4_gptq(W, X, percdamp=0.0)
    assert w4.w4_device_status() == w4.W4_OK


def test_full_size_sampled_rows():
    """The qkv projection of a 7B layer (12288 x 4096) with 512 calibration
    rows: the column loop on the whole layer given the oracle's U, 64 sampled
    rows bit-equal; then the whole pipeline: its U within tolerance of the
    oracle's fp64 factor, 64 sampled rows bit-equal to the oracle's column
    loop on that U, and its calibration error below RTN's (computed on the
    device with PyTorch)."""
    c = synth.GPTQ
    N, K, Mc = c["N"], c["K"], c["Mc"]
    W = synth.weights(N, K, c["std"], c["seed"], outlier_frac=c["w_outlier"], dtype=c["dtype"])
    X = synth.activations(Mc, K, c["seed"], salient_frac=c["x_salient"], dtype=c["dtype"])
    Uo = oracle.gptq_inverse_factor(oracle.gptq_hessian(bits(X), odt(X)), c["percdamp"])
    U32 = Uo.astype(np.float32)
    Wd, Xd = W.to(DEV), X.to(DEV)
    p, s, z = w4.w4_gptq_quantize(Wd, torch.from_numpy(U32).to(DEV), sym=c["sym"])
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(2).choice(N, 64, replace=False))
    po, so, zo = oracle.gptq_quantize(bits(W)[rows], odt(W), U32, 128, c["sym"])
    assert np.array_equal(p.cpu().numpy()[rows], po)
    assert np.array_equal(s.cpu().numpy()[rows], so)
    assert np.array_equal(z.cpu().numpy()[rows], zo)
    p2, s2, z2, U = w4.w4_gptq(Wd, Xd, sym=c["sym"], percdamp=c["percdamp"], return_u=True)
    torch.cuda.synchronize()
    Ug32 = U.cpu().numpy()
    assert np.abs(Ug32.astype(np.float64) - Uo).max() <= 2e-3 * np.abs(Uo).max()
    po2, so2, zo2 = oracle.gptq_quantize(bits(W)[rows], odt(W), Ug32, 128, c["sym"])
    assert np.array_equal(p2.cpu().numpy()[rows], po2)
    assert np.array_equal(s2.cpu().numpy()[rows], so2)
    assert np.array_equal(z2.cpu().numpy()[rows], zo2)
    # calibration error on the device (plain PyTorch), GPTQ vs RTN
    def err(pk, sc, zp):
        codes = torch.stack([(pk.int() >> sh) & 15 for sh in (0, 4)], -1).reshape(N, K // 8, 4, 2)
        # word j = bytes 4j..4j+3; byte b holds nibbles 2b (low) and 2b+1 (high);
        # nibble i holds k = 8j + {0,2,4,6,1,3,5,7}[i]
        nib = codes.reshape(N, K // 8, 8)
        order = torch.tensor([0, 4, 1, 5, 2, 6, 3, 7], device=DEV)
        u = nib[:, :, order].reshape(N, K).float()
        deq = (u - zp.repeat_interleave(128, 1)) * sc.repeat_interleave(128, 1)
        return torch.linalg.norm((deq.double() - Wd.double()) @ Xd.double().T).item()
    pr, sr, zr = w4.w4_quantize(Wd, 128, sym=c["sym"])
    e_g, e_r = err(p2, s2, z2), err(pr, sr, zr)
    assert e_g < 0.8 * e_r, (e_g, e_r)
    assert w4.w4_device_status() == w4.W4_OK
