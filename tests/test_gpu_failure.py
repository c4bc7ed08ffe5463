"""Failure detection on the GPU without a GPU fault.

Every wait in the library's kernels is bounded: when one runs out the kernel
sets the device status word, leaves its loops, drains what it has in flight
and returns, so the context stays usable.  `w4_selftest_wait_timeout`
enqueues a kernel whose only wait can never complete, with a short bound;
these tests check that the status word reports it, that reading it with
reset clears it, and that the layer still computes correct results after.
"""
import ctypes

import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gemm_matches_oracle(M, N, K, seed):
    W = synth.weights(N, K, 0.02, seed)
    X = synth.activations(M, K, seed)
    packed, scales, zeros = oracle_quantize(W, 128, False)
    pd = torch.from_numpy(packed).to(DEV)
    sd = torch.from_numpy(scales).to(DEV)
    zd = torch.from_numpy(zeros).to(DEV)
    Y = w4.w4a16_gemm(X.to(DEV), pd, sd, zd)
    torch.cuda.synchronize()
    check_y(Y, oracle_linear(X, packed, scales, zeros, K, 128), f"after timeout M={M}")


def test_wait_timeout_sets_status_and_context_survives():
    assert w4.w4_device_status(reset=True) in (w4.W4_OK, w4.W4_ERR_TIMEOUT)
    assert w4.w4_device_status() == w4.W4_OK
    w4.w4_selftest_wait_timeout(2000)  # 2 ms
    assert w4.w4_device_status(reset=True) == w4.W4_ERR_TIMEOUT
    assert w4.w4_device_status() == w4.W4_OK  # cleared by the reset above
    # the context is still usable: decode and prefill paths give correct results
    _gemm_matches_oracle(1, 1000, 1024, 11)
    _gemm_matches_oracle(200, 300, 512, 12)
    assert w4.w4_device_status() == w4.W4_OK


def test_timeout_is_bounded_by_its_limit():
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    w4.w4_selftest_wait_timeout(5000)  # 5 ms
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    assert 4.0 <= ms < 500.0, ms
    assert w4.w4_device_status(reset=True) == w4.W4_ERR_TIMEOUT


def test_selftest_rejects_out_of_range_timeouts():
    lib = w4.load()
    for bad in (0, 1000001):
        assert lib.w4_selftest_wait_timeout(bad, None) == w4.W4_ERR_INVALID_ARG
    assert w4.w4_device_status() == w4.W4_OK
