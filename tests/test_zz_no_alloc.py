"""w4a16_gemm_noalloc: the decode layer for callers that cannot allocate
device memory (its scratch space is a fixed array inside the library).

Called through the C ABI and compared with w4a16_gemm on the same inputs,
within the W4A16 tolerance of the other parity tests, on two calls in a row.
This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes alone in a fresh process."""
import ctypes

import pytest
import torch

import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(N, K, sym, seed):
    W = synth.weights(N, K, 0.02, seed, outlier_frac=0.001).to(DEV)
    return w4.w4_quantize(W, 128, sym=sym)


@pytest.mark.parametrize("M,N,K,sym", [(1, 512, 8192, False), (8, 1000, 4096, True),
                                       (3, 11008, 4096, False)])
def test_matches_w4a16_gemm_on_two_calls(M, N, K, sym):
    packed, scales, zeros = _layer(N, K, sym, 7 + M)
    for call in range(2):
        X = synth.activations(M, K, 100 * call + M, salient_frac=0.01).to(DEV)
        ref = w4.w4a16_gemm(X, packed, scales, zeros)
        got = w4.w4a16_gemm_noalloc(X, packed, scales, zeros)
        torch.cuda.synchronize()
        check_y(got, ref.double().cpu().numpy(), f"no-alloc call {call}")
    assert w4.w4_device_status() == w4.W4_OK


def test_through_raw_c_abi():
    lib = w4.load()
    M, N, K = 2, 384, 8192
    packed, scales, zeros = _layer(N, K, False, 3)
    X = synth.activations(M, K, 3).to(DEV)
    Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    st = lib.w4a16_gemm_noalloc(ctypes.c_void_p(X.data_ptr()), w4.W4_F16, M,
                                ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                ctypes.c_void_p(zeros.data_ptr()), K, N, 128,
                                ctypes.c_void_p(Y.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == w4.W4_OK
    ref = w4.w4a16_gemm(X, packed, scales, zeros)
    torch.cuda.synchronize()
    check_y(Y, ref.double().cpu().numpy(), "raw C ABI")


def test_rejects_what_it_cannot_serve():
    M, N, K = 64, 256, 1024
    packed, scales, zeros = _layer(N, K, False, 5)
    X = synth.activations(M, K, 5).to(DEV)
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemm_noalloc(X, packed, scales, zeros)
    assert e.value.status == w4.W4_ERR_UNSUPPORTED
    # a shape whose workspace exceeds the 4 MiB array, when this GPU plans one
    M, N, K = 32, 25600, 8192
    if w4.w4a16_workspace_bytes(M, K, N) > (4 << 20):
        lib = w4.load()
        st = lib.w4a16_gemm_noalloc(ctypes.c_void_p(16), w4.W4_F16, M, ctypes.c_void_p(16),
                                    ctypes.c_void_p(16), None, K, N, 128, ctypes.c_void_p(16),
                                    None)
        assert st == w4.W4_ERR_UNSUPPORTED
        assert "4 MiB" in w4.w4_last_error()
