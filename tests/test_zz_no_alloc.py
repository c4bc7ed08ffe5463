"""w4a16_gemm_noalloc: the decode layer for callers that cannot allocate
device memory (its scratch space is a fixed array inside the library).

Called through the C ABI on shapes whose decode kernel does use scratch
space, and checked two ways on two calls in a row, with a call of another
shape in between (so the array holds another call's leftovers):
  * against the oracle's fp64 product, within the W4A16 tolerance of the
    other parity tests;
  * bit for bit against w4a16_gemm on the same inputs (the same kernel with a
    caller-provided workspace; its reduction order is fixed).
This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes alone in a fresh process."""
import ctypes

import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(N, K, sym, seed):
    W = synth.weights(N, K, 0.02, seed, outlier_frac=0.001)
    p, s, z = oracle_quantize(W, 128, sym)
    dev = tuple(torch.from_numpy(a).to(DEV) for a in (p, s, z))
    return (p, s, z), dev


def _raw_noalloc(X, packed, scales, zeros, Y):
    lib = w4.load()
    M, K = X.shape
    N = packed.shape[0]
    return lib.w4a16_gemm_noalloc(ctypes.c_void_p(X.data_ptr()), w4.W4_F16, M,
                                  ctypes.c_void_p(packed.data_ptr()),
                                  ctypes.c_void_p(scales.data_ptr()),
                                  None if zeros is None else ctypes.c_void_p(zeros.data_ptr()),
                                  K, N, 128, ctypes.c_void_p(Y.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K,sym", [(1, 512, 8192, False), (16, 1000, 4096, True),
                                       (24, 11008, 4096, False)])
def test_matches_oracle_and_w4a16_gemm_on_two_calls(M, N, K, sym):
    assert w4.w4a16_workspace_bytes(M, K, N) > 0, "shape must use scratch space"
    host, (packed, scales, zeros) = _layer(N, K, sym, 7 + M)
    # another shape, run in between, leaves its own contents in the array
    o_host, (op, os_, oz) = _layer(300, 8192, False, 99)
    Xo = synth.activations(5, 8192, 99).to(DEV)
    for call in range(2):
        X = synth.activations(M, K, 100 * call + M, salient_frac=0.01)
        Xd = X.to(DEV)
        got = torch.empty((M, N), dtype=torch.float16, device=DEV)
        assert _raw_noalloc(Xd, packed, scales, zeros, got) == w4.W4_OK
        ref = w4.w4a16_gemm(Xd, packed, scales, zeros)
        torch.cuda.synchronize()
        check_y(got, oracle_linear(X, *host, K), f"no-alloc call {call}")
        assert torch.equal(got, ref), f"call {call}: differs from w4a16_gemm"
        Yo = torch.empty((5, 300), dtype=torch.float16, device=DEV)
        assert _raw_noalloc(Xo, op, os_, oz, Yo) == w4.W4_OK
        torch.cuda.synchronize()
    assert w4.w4_device_status() == w4.W4_OK


def test_rejects_what_it_cannot_serve():
    M, N, K = 64, 256, 1024
    _, (packed, scales, zeros) = _layer(N, K, False, 5)
    X = synth.activations(M, K, 5).to(DEV)
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemm_noalloc(X, packed, scales, zeros)
    assert e.value.status == w4.W4_ERR_UNSUPPORTED
    # a shape whose workspace exceeds the 4 MiB array, when this GPU plans
    # one: rejected before any launch (the buffers are real, so even a
    # regression of that check would only compute a result)
    M, N, K = 32, 25600, 8192
    if w4.w4a16_workspace_bytes(M, K, N) > (4 << 20):
        X = torch.zeros((M, K), dtype=torch.float16, device=DEV)
        packed = torch.zeros((N, K // 2), dtype=torch.uint8, device=DEV)
        scales = torch.zeros((N, K // 128), dtype=torch.float32, device=DEV)
        Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
        assert _raw_noalloc(X, packed, scales, None, Y) == w4.W4_ERR_UNSUPPORTED
        assert "4 MiB" in w4.w4_last_error()
