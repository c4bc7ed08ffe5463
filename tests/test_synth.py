"""The seeded input generator: reproducible, and shaped like the workloads' recipe."""
import math

import torch

import synth


def test_splitmix64_reference_values():
    # SplitMix64 with state 0: the first outputs of the published generator
    # (Steele, Lea & Flood 2014; also java.util.SplittableRandom with seed 0)
    got = synth.raw64(0, 0, 3)
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [int(v) & ((1 << 64) - 1) for v in got] == want


def test_deterministic_and_chunk_independent():
    a = synth.weights(64, 256, 0.02, seed=9, outlier_frac=0.01)
    b = synth.weights(64, 256, 0.02, seed=9, outlier_frac=0.01, chunk_rows=7)
    assert torch.equal(a, b)
    c = synth.weights(64, 256, 0.02, seed=10, outlier_frac=0.01)
    assert not torch.equal(a, c)


def test_weight_distribution():
    W = synth.weights(512, 1024, 0.02, seed=2, outlier_frac=0.001).double()
    big = W.abs() > 0.02 * 6
    frac = big.double().mean().item()
    assert 0.0004 < frac < 0.0016  # ~0.1% entries x10 (plus a few 6-sigma draws)
    core = W[~big]
    assert abs(core.mean().item()) < 1e-3
    assert abs(core.std().item() - 0.02) < 1e-3


def test_salient_channels():
    K = 4096
    ch = synth.salient_channels(K, 0.01, seed=2)
    assert ch.numel() == math.floor(0.01 * K) == 40
    assert ch.unique().numel() == 40
    X = synth.activations(256, K, seed=2, salient_frac=0.01).double()
    colstd = X.std(dim=0)
    assert (colstd[ch] > 10).all()
    mask = torch.ones(K, dtype=torch.bool)
    mask[ch] = False
    assert (colstd[mask] < 2).all()


def test_bf16_and_awq_scale():
    X = synth.activations(512, 256, seed=5, salient_frac=0.02, dtype="bf16")
    assert X.dtype == torch.bfloat16
    s = synth.awq_col_scale(X)
    assert s.dtype == torch.float32 and s.shape == (256,)
    ch = synth.salient_channels(256, 0.02, seed=5)
    assert (s[ch] > 3).all()
