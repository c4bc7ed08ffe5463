"""The C ABI of libw4a16.so, checked without a GPU: it builds, loads, exports
every function include/w4a16.h declares, and rejects invalid arguments with
the documented status before anything reaches the device.

The argument checks pass fake, never-dereferenced addresses.  They only ever
run in a process that sees no GPU: where a GPU is visible, this module's tests
are skipped in-process and re-run as a child pytest with
CUDA_VISIBLE_DEVICES="", so that even a regression in the host-side checks
could not launch a kernel on those addresses (the call would fail with
W4_ERR_CUDA instead)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import weight_only_int4_pack_b200 as w4
from weight_only_int4_pack_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _gpu_visible():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


GPU_VISIBLE = _gpu_visible()


@pytest.fixture(autouse=True)
def _no_visible_gpu(request):
    if GPU_VISIBLE and request.node.name != "test_module_in_a_process_without_gpu":
        pytest.skip("fake-address checks run in a child process without a visible GPU")


@pytest.mark.skipif(not GPU_VISIBLE, reason="runs in-process here: no GPU is visible")
def test_module_in_a_process_without_gpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.abspath(__file__)], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return w4.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(w4\w*)\s*\(", src, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("w4_quantize", "w4a16_gemm", "w4a16_workspace_bytes", "w4_status_string",
                 "w4_device_status", "w4_abi_version"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings(lib):
    assert w4.w4_abi_version() == 0x00010003
    assert w4.w4_status_string(0) == "W4_OK"
    assert w4.w4_status_string(1) == "W4_ERR_INVALID_ARG"
    assert w4.w4_status_string(2) == "W4_ERR_UNSUPPORTED"
    assert w4.w4_status_string(3) == "W4_ERR_CUDA"
    assert w4.w4_status_string(4) == "W4_ERR_TIMEOUT"
    assert w4.w4_status_string(5) == "W4_ERR_BOUNDS"
    assert w4.w4_status_string(99) == "W4_ERR_UNKNOWN"


# Fake, 16-byte aligned, never-dereferenced addresses: validation must reject
# before any of them is touched.
A = ctypes.c_void_p(0x100000)
B = ctypes.c_void_p(0x200000)
C = ctypes.c_void_p(0x300000)
D = ctypes.c_void_p(0x400000)
S = ctypes.c_void_p(0)


@pytest.mark.parametrize("args,status", [
    # (W, wt, K, N, group, sym, col_scale, packed, scales, zeros)
    ((A, 0, 192, 4, 128, 1, None, B, C, D), 1),    # K % group != 0 (the pages' assert)
    ((A, 0, 0, 4, 128, 1, None, B, C, D), 1),      # K == 0
    ((A, 0, 256, -1, 128, 1, None, B, C, D), 1),   # N < 0
    ((A, 2, 256, 4, 128, 1, None, B, C, D), 1),    # bad dtype
    ((A, 0, 256, 4, 0, 1, None, B, C, D), 1),      # group 0
    ((None, 0, 256, 4, 128, 1, None, B, C, D), 1), # null W
    ((A, 0, 256, 4, 128, 1, None, None, C, D), 1), # null packed
    ((A, 0, 256, 4, 128, 1, None, B, None, D), 1), # null scales
    ((A, 0, 256, 4, 128, 1, None, B, C, None), 1), # null zeros
    ((A, 0, 132, 4, 4, 1, None, B, C, D), 1),      # K % 8 != 0
    ((A, 0, 384, 4, 96, 1, None, B, C, D), 2),     # group not in {32,64,128,256}
    ((A, 0, 512, 4, 512, 1, None, B, C, D), 2),
    ((ctypes.c_void_p(0x100008), 0, 256, 4, 128, 1, None, B, C, D), 2),  # misaligned W
    ((A, 0, 256, 4, 128, 1, ctypes.c_void_p(0x500004), B, C, D), 2),     # misaligned col_scale
    ((A, 0, 256, 0, 128, 1, None, None, None, None), 0),  # N == 0: nothing to do
])
def test_quantize_argument_checks(lib, args, status):
    assert lib.w4_quantize(*args, S) == status


@pytest.mark.parametrize("args,status", [
    # (X, xt, M, packed, scales, zeros, K, N, group, Y, ws, ws_bytes)
    ((A, 0, 1, B, C, None, 192, 8, 128, D, None, 0), 1),   # K % group
    ((A, 0, -1, B, C, None, 256, 8, 128, D, None, 0), 1),   # M < 0
    ((A, 0, 1, B, C, None, 256, -3, 128, D, None, 0), 1),   # N < 0
    ((A, 0, 1, B, C, None, 0, 8, 128, D, None, 0), 1),      # K == 0
    ((A, 5, 1, B, C, None, 256, 8, 128, D, None, 0), 1),    # dtype
    ((None, 0, 1, B, C, None, 256, 8, 128, D, None, 0), 1), # null X
    ((A, 0, 1, None, C, None, 256, 8, 128, D, None, 0), 1), # null packed
    ((A, 0, 1, B, None, None, 256, 8, 128, D, None, 0), 1), # null scales
    ((A, 0, 1, B, C, None, 256, 8, 128, None, None, 0), 1), # null Y
    ((A, 0, 1, B, C, None, 256, 8, 64, D, None, 0), 2),     # only group 128 multiplies
    ((A, 0, 1, ctypes.c_void_p(0x200004), C, None, 256, 8, 128, D, None, 0), 2),  # misaligned
    ((A, 0, 0, B, C, None, 256, 8, 128, D, None, 0), 0),    # M == 0: nothing to do
    ((A, 0, 4, B, C, None, 256, 0, 128, D, None, 0), 0),    # N == 0: nothing to do
])
def test_gemm_argument_checks(lib, args, status):
    assert lib.w4a16_gemm(*args, S) == status


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(w4, "lib_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(w4, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        w4.load()


def test_product_package_does_not_reach_the_oracle():
    pkg = os.path.join(ROOT, "weight_only_int4_pack_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if not fn.endswith((".py", ".cu", ".cuh", ".h")):
                continue
            src = open(os.path.join(dirpath, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn
            assert "w4ref" not in src and "libw4ref" not in src, fn


def test_selftest_argument_check(lib):
    """The timeout range is checked on the host before any CUDA call."""
    for bad in (0, 1000001):
        assert lib.w4_selftest_wait_timeout(bad, None) == w4.W4_ERR_INVALID_ARG
        assert b"timeout_us" in lib.w4_last_error()


ALPHAS = (ctypes.c_float * 3)(0.0, 0.5, 1.0)
BAD_ALPHAS = (ctypes.c_float * 2)(0.0, 1.5)
E = ctypes.c_void_p(0x600000)
F = ctypes.c_void_p(0x700000)
WS = ctypes.c_void_p(0x10000000)


@pytest.mark.parametrize("args,status", [
    # (W, X, xt, Mc, K, N, group, sym, alphas, n_alpha, err, best_scale, best_index,
    #  packed_out, scales_out, zeros_out, ws, ws_bytes)
    ((A, B, 0, 16, 192, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 1),  # K % 128
    ((A, B, 0, 0, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 1),   # Mc 0
    ((A, B, 0, 16, 256, 0, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 1),   # N 0
    ((A, B, 7, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 1),  # dtype
    ((A, B, 0, 16, 256, 64, 64, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 2),   # group
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 0, C, D, E, None, None, None, WS, 1 << 30), 1),  # none
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 65, C, D, E, None, None, None, WS, 1 << 30), 1), # > 64
    ((A, B, 0, 16, 256, 64, 128, 0, BAD_ALPHAS, 2, C, D, E, None, None, None, WS, 1 << 30), 1),
    ((A, B, 0, 16, 256, 64, 128, 0, None, 3, C, D, E, None, None, None, WS, 1 << 30), 1),
    ((None, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1 << 30), 1),
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, None, D, E, None, None, None, WS, 1 << 30), 1),
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, None, None, None, None, WS, 1 << 30), 1),
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, F, None, None, WS, 1 << 30), 1),     # partial q
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None, WS, 1024), 1),     # ws small
    ((A, B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None,
      ctypes.c_void_p(0x10000010), 1 << 30), 1),                                             # ws align
    ((ctypes.c_void_p(0x100004), B, 0, 16, 256, 64, 128, 0, ALPHAS, 3, C, D, E, None, None, None,
      WS, 1 << 30), 2),                                                                      # W align
])
def test_awq_search_argument_checks(lib, args, status):
    assert lib.w4_awq_search(*args, S) == status


def test_awq_search_workspace_size(lib):
    Mc, K, N = 512, 4096, 12288
    need = w4.w4_awq_search_workspace_bytes(Mc, K, N)
    floor = N * K // 2 + 2 * N * (K // 128) * 4 + 2 * Mc * K + 2 * Mc * N + 4 * Mc * N
    assert floor <= need <= floor + 48 * 8 * K + 64 * 1024
    assert w4.w4_awq_search_workspace_bytes(Mc, 4000, N) == 0   # K % 128
    assert w4.w4_awq_search_workspace_bytes(0, K, N) == 0
    assert w4.w4_awq_search_workspace_bytes(16, K, N) >= w4.w4a16_workspace_bytes(16, K, N)


@pytest.mark.parametrize("args,status", [
    # (A, at, rows, K, col, col_op, fmt, q, scale)
    ((A, 0, 4, 40, None, 0, 0, B, C), 1),      # K % 16
    ((A, 0, 0, 64, None, 0, 0, B, C), 1),      # rows 0
    ((A, 3, 4, 64, None, 0, 0, B, C), 1),      # dtype
    ((A, 0, 4, 64, None, 0, 2, B, C), 1),      # fmt
    ((A, 0, 4, 64, None, 3, 0, B, C), 1),      # col_op
    ((A, 0, 4, 64, None, 1, 0, B, C), 1),      # col missing for W8_COL_MUL
    ((None, 0, 4, 64, None, 0, 0, B, C), 1),
    ((A, 0, 4, 64, None, 0, 0, None, C), 1),
    ((A, 0, 4, 64, None, 0, 0, B, None), 1),
    ((ctypes.c_void_p(0x100008), 0, 4, 64, None, 0, 0, B, C), 2),  # misaligned A
    ((A, 0, 4, 64, None, 0, 0, B, ctypes.c_void_p(0x300004)), 2),  # misaligned scale
])
def test_w8_quantize_argument_checks(lib, args, status):
    assert lib.w8_quantize(*args, S) == status


@pytest.mark.parametrize("args,status", [
    # (Xq, x_scale, Wq, w_scale, fmt, M, K, N, Y, yt)
    ((A, B, C, D, 0, 4, 40, 8, E, 0), 1),      # K % 16
    ((A, B, C, D, 0, 0, 64, 8, E, 0), 1),      # M 0
    ((A, B, C, D, 0, 4, 64, 0, E, 0), 1),      # N 0
    ((A, B, C, D, 5, 4, 64, 8, E, 0), 1),      # fmt
    ((A, B, C, D, 0, 4, 64, 8, E, 9), 1),      # out dtype
    ((A, B, C, D, 0, 4, 140000, 8, E, 0), 2),  # INT8 accumulator range
    ((A, None, C, D, 0, 4, 64, 8, E, 0), 1),
    ((A, B, C, D, 0, 4, 64, 8, None, 0), 1),
    ((A, B, ctypes.c_void_p(0x300008), D, 0, 4, 64, 8, E, 0), 2),
])
def test_w8_gemm_argument_checks(lib, args, status):
    assert lib.w8_gemm(*args, S) == status


def test_w8_smooth_and_linear_argument_checks(lib):
    F = ctypes.c_float
    # (X, W, xt, Mc, K, N, alpha, s, ws, ws_bytes)
    assert lib.w8_smooth_scales(A, B, 0, 8, 64, 16, F(1.5), C, WS, 8 * 64, S) == 1
    assert lib.w8_smooth_scales(A, B, 0, 8, 64, 16, F(0.5), C, WS, 8 * 63, S) == 1
    assert lib.w8_smooth_scales(A, B, 0, 8, 40, 16, F(0.5), C, WS, 8 * 64, S) == 1
    assert lib.w8_smooth_scales(A, B, 0, 0, 64, 16, F(0.5), C, WS, 8 * 64, S) == 1
    assert lib.w8_smooth_scales(A, None, 0, 8, 64, 16, F(0.5), C, WS, 8 * 64, S) == 1
    assert w4.w8a8_workspace_bytes(3, 64) == 512
    assert w4.w8a8_workspace_bytes(3, 40) == 0
    # (X, xt, M, K, s, fmt, Wq, w_scale, N, Y, ws, ws_bytes)
    assert lib.w8a8_linear(A, 0, 3, 64, None, 0, B, C, 8, D, WS, 256, S) == 1   # small ws
    assert lib.w8a8_linear(A, 0, 3, 64, None, 0, B, C, 8, D,
                           ctypes.c_void_p(0x10000010), 512, S) == 2            # ws align
    assert lib.w8a8_linear(A, 0, 3, 64, None, 0, B, C, 0, D, WS, 512, S) == 1   # N 0


def test_gptq_argument_checks(lib):
    F = ctypes.c_float
    # (W, X, xt, Mc, K, N, group, sym, percdamp, packed, scales, zeros, U_out, ws, ws_bytes)
    ok = (A, B, 0, 64, 256, 32, 128, 0, F(0.01), C, D, E, None, WS, 1 << 30)
    def call(**kw):
        a = list(ok)
        names = ["W", "X", "xt", "Mc", "K", "N", "group", "sym", "pd", "p", "s", "z", "U", "ws",
                 "wsb"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.w4_gptq(*a, S)
    assert call(K=192) == 1            # K % 128
    assert call(group=64) == 2         # group must be 128
    assert call(Mc=0) == 1
    assert call(N=0) == 1
    assert call(N=65535 * 128 + 1) == 1   # beyond the lazy update's grid
    assert call(xt=4) == 1
    assert call(pd=F(-0.5)) == 1
    assert call(W=None) == 1
    assert call(wsb=1024) == 1
    assert call(ws=ctypes.c_void_p(0x10000010)) == 1
    assert call(X=ctypes.c_void_p(0x200008)) == 2
    need = w4.w4_gptq_workspace_bytes(64, 256, 32)
    assert need >= 4 * 256 * 256 + 4 * 32 * 256
    assert w4.w4_gptq_workspace_bytes(64, 200, 32) == 0
    q = w4.w4_gptq_quantize_workspace_bytes(256, 32)
    assert 4 * 32 * 256 + 512 * 32 <= q < need
    # (W, wt, K, N, group, sym, U, packed, scales, zeros, ws, ws_bytes)
    assert lib.w4_gptq_quantize(A, 0, 256, 32, 128, 0, None, C, D, E, WS, q, S) == 1
    assert lib.w4_gptq_quantize(A, 0, 256, 32, 128, 0, B, C, D, E, WS, q - 1, S) == 1
    assert lib.w4_gptq_quantize(A, 0, 256, 32, 32, 0, B, C, D, E, WS, q, S) == 2
