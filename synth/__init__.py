"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds no quantization arithmetic: it only draws numbers.  Both the
CUDA path and the CPU oracle receive the very tensors made here.

Generators (both published methods, written out here):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014), used in counter form: draw i of a stream with
    key s is mix(s + (i + 1) * 0x9E3779B97F4A7C15).
  * Box-Muller (1958): z = sqrt(-2 ln u1) * cos(2 pi u2), u from the top 53 bits.

All integer work is done in torch int64, whose multiply wraps modulo 2^64; a
logical right shift is an arithmetic shift followed by a mask.  The same code
runs on CPU (tests) and on a CUDA device (large benchmark inputs).  The float
part (log, cos in fp64) may differ in the last ulp between the two devices;
tests therefore always draw on one device and copy.

Input recipe of the workloads (weights [out][in] = [N][K], activations [M][K]):
  * weights: N(0, std) rounded once to fp16/bf16, with a Bernoulli(frac) mask
    of entries multiplied by 10 before rounding ("0.1% entries x10");
  * activations: N(0, 1) with floor(frac * K) distinct input channels (the K
    smallest hash values of a dedicated stream) multiplied by 20;
  * AWQ column factor of the 7B-stack workload: s_j = (mean_i |Xcal_ij|)^0.5
    over a calibration batch, in fp64, rounded once to fp32.
"""
from __future__ import annotations

import math

import torch

_GAMMA = -7046029254386353131  # 0x9E3779B97F4A7C15 as int64
_M1 = -4658895280553007687  # 0xBF58476D1CE4E5B9
_M2 = -7723592293110705685  # 0x94D049BB133111EB


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _M1
    z = (z ^ _lsr(z, 27)) * _M2
    return z ^ _lsr(z, 31)


def _to_i64(v: int) -> int:
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def stream_key(seed: int, tensor_id: int) -> int:
    """A distinct SplitMix64 key per (seed, tensor) pair."""
    t = torch.tensor([_to_i64(seed * 16 + tensor_id)], dtype=torch.int64)
    return int(_mix(t + _GAMMA)[0])


def raw64(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Draws start..start+count-1 of the SplitMix64 stream `key` (int64 bit patterns)."""
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix(i * _GAMMA + key)


def uniform(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """U[0,1) doubles from the top 53 bits of each draw."""
    return _lsr(raw64(key, start, count, device), 11).to(torch.float64) * (2.0 ** -53)


def normal(key: int, count: int, device="cpu", chunk: int = 1 << 26) -> torch.Tensor:
    """N(0,1) doubles by Box-Muller; normal i uses draws 2i and 2i+1."""
    out = torch.empty(count, dtype=torch.float64, device=device)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        u = uniform(key, 2 * c0, 2 * n, device).view(n, 2)
        r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))  # 1 - u1 lies in (0, 1]
        out[c0:c0 + n] = r * torch.cos((2.0 * math.pi) * u[:, 1])
    return out


def _dtype(name):
    return {"f16": torch.float16, "fp16": torch.float16, "bf16": torch.bfloat16,
            torch.float16: torch.float16, torch.bfloat16: torch.bfloat16}[name]


def weights(N: int, K: int, std: float, seed: int, outlier_frac: float = 0.0,
            outlier_mult: float = 10.0, dtype="f16", device="cpu", tensor_id: int = 0,
            chunk_rows: int = 4096) -> torch.Tensor:
    """W [N][K] ~ N(0, std), a Bernoulli(outlier_frac) subset of entries x outlier_mult."""
    key = stream_key(seed, tensor_id)
    okey = stream_key(seed, tensor_id + 8)
    dt = _dtype(dtype)
    W = torch.empty((N, K), dtype=dt, device=device)
    thresh = int(outlier_frac * 2.0 ** 53)
    for r0 in range(0, N, chunk_rows):
        nr = min(chunk_rows, N - r0)
        # each row block draws its own slice of the stream so the result is
        # independent of chunk_rows
        v = _normal_slice(key, r0 * K, nr * K, device) * std
        if outlier_frac > 0:
            sel = _lsr(raw64(okey, r0 * K, nr * K, device), 11) < thresh
            v = torch.where(sel, v * outlier_mult, v)
        W[r0:r0 + nr] = v.view(nr, K).to(dt)
    return W


def _normal_slice(key: int, start: int, count: int, device) -> torch.Tensor:
    u = uniform(key, 2 * start, 2 * count, device).view(count, 2)
    r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
    return r * torch.cos((2.0 * math.pi) * u[:, 1])


def salient_channels(K: int, frac: float, seed: int, tensor_id: int = 3) -> torch.Tensor:
    """floor(frac*K) distinct channel indices: the smallest hash values of a stream."""
    n = int(math.floor(frac * K))
    if n == 0:
        return torch.zeros(0, dtype=torch.int64)
    h = _lsr(raw64(stream_key(seed, tensor_id), 0, K), 1)
    return torch.sort(torch.argsort(h)[:n]).values


def activations(M: int, K: int, seed: int, salient_frac: float = 0.0, salient_mult: float = 20.0,
                dtype="f16", device="cpu", tensor_id: int = 1) -> torch.Tensor:
    """X [M][K] ~ N(0,1); floor(salient_frac*K) input channels x salient_mult."""
    dt = _dtype(dtype)
    v = _normal_slice(stream_key(seed, tensor_id), 0, M * K, device).view(M, K)
    ch = salient_channels(K, salient_frac, seed).to(device)
    if ch.numel():
        v[:, ch] *= salient_mult
    return v.to(dt)


def awq_col_scale(Xcal: torch.Tensor) -> torch.Tensor:
    """Column factor s_j = (mean_i |Xcal_ij|)^0.5 in fp64, rounded once to fp32."""
    return Xcal.to(torch.float64).abs().mean(dim=0).sqrt().to(torch.float32)


# ---- the workloads ----------------------------------------------------------------------

TINY = dict(name="tiny", N=256, K=512, M=1, std=0.02, seed=0, sym=True, dtype="f16")
DECODE_M1 = dict(name="decode_m1", K=4096, Ns=(4096, 11008, 12288), M=1, std=0.02, seed=2,
                 sym=False, dtype="f16", w_outlier=0.001, x_salient=0.01)
DECODE_SMALLM = dict(name="decode_small_m", K=8192, N=28672, Ms=(4, 8, 16, 32), std=0.015,
                     seed=3, sym=True, dtype="f16", x_salient=0.01)
PREFILL = dict(name="prefill", M=2048, K=4096, N=11008, std=0.02, seed=4, sym=False,
               dtype="bf16", x_salient=0.01)
# (out, in) of the four projections of one 7B layer; 32 layers
STACK_7B = dict(name="quant_7b_stack", layers=32,
                shapes=(("qkv", 12288, 4096), ("o", 4096, 4096), ("gate_up", 22016, 4096),
                        ("down", 4096, 11008)),
                std=0.02, seed=5, sym=False, dtype="f16", w_outlier=0.001, calib_M=512,
                x_salient=0.01)
# AWQ alpha search on one 7B projection (qkv, 12288 x 4096) with 512 calibration rows
AWQ_SEARCH = dict(name="awq_search", Mc=512, K=4096, N=12288, n_alpha=11, std=0.02, seed=6,
                  sym=False, dtype="f16", w_outlier=0.001, x_salient=0.01)
# W8A8 layer (SmoothQuant INT8 / FP8 E4M3) on the prefill shape
W8A8 = dict(name="w8a8", M=2048, K=4096, N=11008, std=0.02, seed=7, dtype="bf16",
            x_salient=0.01, alpha=0.5)
# GPTQ on one 7B projection (qkv, 12288 x 4096) with 512 calibration rows
GPTQ = dict(name="gptq", N=12288, K=4096, Mc=512, std=0.02, seed=8, dtype="f16", sym=False,
            w_outlier=0.001, x_salient=0.01, percdamp=0.01)
