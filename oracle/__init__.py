"""CPU oracle for per-group INT4 RTN quantization and the W4A16 linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
CPU-baseline leg of the benchmark may import this package; the CUDA library
never does, and the two share no code.  The arithmetic lives in ``w4ref.c``
(plain scalar C, fp32 IEEE quantizer, fp64 dequantization and matmul); this
module only builds it with gcc and marshals numpy arrays through ctypes.

Sources followed (see ``w4ref.c`` for the step-by-step citations):
"LLM quantization methods: principles and implementation"
(zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3 and §4.2, and
"PTQ weight quantization: from GPTQ to AWQ" (jonathanding.github.io),
sections "Round-to-Nearest" and "AWQ" (the AWQ scale search of §4.2 is
``awq_search``); §4.3 SmoothQuant and §4.6 FP8 for the W8A8 layer
(``smooth_scales``, ``quant8``, ``gemm8``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4ref.c")
_LIB = os.path.join(_HERE, "libw4ref.so")

F16 = 0
BF16 = 1
INT8 = 0
E4M3 = 1

OK = 0
EINVAL = 1
ENONFINITE = 5

_lib = None


def build(force: bool = False) -> str:
    """Compile w4ref.c into libw4ref.so next to it (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        lib.w4ref_quantize.argtypes = [P, I, L, L, L, I, P, P, P, P]
        lib.w4ref_quantize.restype = I
        lib.w4ref_dequant.argtypes = [P, P, P, L, L, L, P]
        lib.w4ref_dequant.restype = I
        lib.w4ref_linear.argtypes = [P, I, L, L, P, L, P, L, P]
        lib.w4ref_linear.restype = I
        lib.w4ref_linear_at.argtypes = [P, I, L, P, P, P, L, L, L]
        lib.w4ref_linear_at.restype = ctypes.c_double
        lib.w4ref_code.argtypes = [P, L, L, L]
        lib.w4ref_code.restype = I
        lib.w4ref_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.w4ref_f16_to_f64.restype = ctypes.c_double
        lib.w4ref_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.w4ref_bf16_to_f64.restype = ctypes.c_double
        lib.w4ref_round16.argtypes = [ctypes.c_double, I]
        lib.w4ref_round16.restype = ctypes.c_double
        lib.w4ref_awq_search.argtypes = [P, P, I, L, L, L, L, I, P, L, P, P, P]
        lib.w4ref_awq_search.restype = I
        lib.w4ref_round_e4m3.argtypes = [ctypes.c_double]
        lib.w4ref_round_e4m3.restype = ctypes.c_double
        lib.w4ref_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.w4ref_e4m3_to_f64.restype = ctypes.c_double
        lib.w4ref_smooth_scales.argtypes = [P, P, I, L, L, L, ctypes.c_double, P]
        lib.w4ref_smooth_scales.restype = I
        lib.w4ref_quant8.argtypes = [P, I, L, L, P, I, I, P, P]
        lib.w4ref_quant8.restype = I
        lib.w4ref_gemm8.argtypes = [P, P, I, L, L, L, ctypes.c_float, ctypes.c_float, I, P, L, P]
        lib.w4ref_gemm8.restype = I
        lib.w4ref_gptq_quantize.argtypes = [P, I, L, L, L, I, P, P, P, P]
        lib.w4ref_gptq_quantize.restype = I
        lib.w4ref_gptq_hessian.argtypes = [P, I, L, L, P]
        lib.w4ref_gptq_hessian.restype = I
        lib.w4ref_threads.argtypes = []
        lib.w4ref_threads.restype = I
        lib.w4ref_set_threads.argtypes = [I]
        lib.w4ref_set_threads.restype = None
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bits16(a: np.ndarray) -> np.ndarray:
    """Accept uint16 bit patterns or np.float16 values; return contiguous uint16 bits."""
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("16-bit inputs are passed as uint16 bit patterns or float16")
    return np.ascontiguousarray(a)


class OracleError(RuntimeError):
    pass


def set_threads(n: int) -> None:
    _load().w4ref_set_threads(int(n))


def threads() -> int:
    return int(_load().w4ref_threads())


def quantize(W, dtype: int, group: int, sym: bool, col_scale=None):
    """Quantize W [N][K] -> (packed uint8 [N][K/2], scales f32 [N][G], zeros f32 [N][G])."""
    W = _bits16(W)
    N, K = W.shape
    if col_scale is not None:
        col_scale = np.ascontiguousarray(col_scale, dtype=np.float32)
        assert col_scale.shape == (K,)
    G = K // group if group > 0 else 0
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, max(G, 1)), np.float32)
    zeros = np.zeros((N, max(G, 1)), np.float32)
    st = _load().w4ref_quantize(_ptr(W), dtype, K, N, group, int(bool(sym)), _ptr(col_scale),
                                _ptr(packed), _ptr(scales), _ptr(zeros))
    if st != OK:
        raise OracleError(f"w4ref_quantize status {st}")
    return packed, scales[:, :G], zeros[:, :G]


def dequant(packed, scales, zeros, K: int, group: int) -> np.ndarray:
    """fp64 W-hat [N][K] = (u - zero) * scale; zeros=None means zero = 8 (symmetric)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    if zeros is not None:
        zeros = np.ascontiguousarray(zeros, dtype=np.float32)
    N = packed.shape[0]
    out = np.empty((N, K), np.float64)
    st = _load().w4ref_dequant(_ptr(packed), _ptr(scales), _ptr(zeros), K, N, group, _ptr(out))
    if st != OK:
        raise OracleError(f"w4ref_dequant status {st}")
    return out


def linear(X, dtype: int, What: np.ndarray, rows=None) -> np.ndarray:
    """fp64 Y = X * W-hat^T (naive loop); rows selects a subset of X's rows."""
    X = _bits16(X)
    M, K = X.shape
    What = np.ascontiguousarray(What, dtype=np.float64)
    N = What.shape[0]
    assert What.shape[1] == K
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rows.shape[0]
    else:
        nr = M
    Y = np.zeros((nr, N), np.float64)
    st = _load().w4ref_linear(_ptr(X), dtype, M, K, _ptr(What), N, _ptr(rows), nr, _ptr(Y))
    if st != OK:
        raise OracleError(f"w4ref_linear status {st}")
    return Y


def linear_at(X, dtype: int, packed, scales, zeros, group: int, pairs) -> np.ndarray:
    """fp64 Y[m][n] for a list of (m, n) pairs, straight from the packed weights."""
    X = _bits16(X)
    M, K = X.shape
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    if zeros is not None:
        zeros = np.ascontiguousarray(zeros, dtype=np.float32)
    lib = _load()
    out = np.empty(len(pairs), np.float64)
    for i, (m, n) in enumerate(pairs):
        out[i] = lib.w4ref_linear_at(_ptr(X), dtype, K, _ptr(packed), _ptr(scales), _ptr(zeros),
                                     group, int(m), int(n))
    return out


def code(packed, K: int, n: int, k: int) -> int:
    """The 4-bit code of weight (n, k) read back from the packed layout."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    return int(_load().w4ref_code(_ptr(packed), K, n, k))


def f16_to_f64(h: int) -> float:
    return float(_load().w4ref_f16_to_f64(h))


def bf16_to_f64(h: int) -> float:
    return float(_load().w4ref_bf16_to_f64(h))


def round16(v: float, dtype: int) -> float:
    """Nearest fp16 / bf16 value to v (ties to even), as a float; +-inf on overflow."""
    return float(_load().w4ref_round16(float(v), dtype))


def awq_search(W, X, dtype: int, group: int, sym: bool, alphas):
    """AWQ grid search over alpha for one layer.

    W [N][K] and calibration activations X [Mc][K] (uint16 bits or float16).
    Returns (err fp64 [n_alpha], s fp32 [n_alpha][K], best index) where
    err[t] = || Q(W * s_t)(X / s_t) - W X ||_F^2 and s_t = (a / w)^alphas[t].
    """
    W = _bits16(W)
    X = _bits16(X)
    N, K = W.shape
    Mc, K2 = X.shape
    assert K2 == K
    alphas = np.ascontiguousarray(alphas, dtype=np.float32).ravel()
    err = np.full(alphas.shape[0], np.nan, np.float64)
    s_all = np.zeros((alphas.shape[0], K), np.float32)
    best = ctypes.c_long(-1)
    st = _load().w4ref_awq_search(_ptr(W), _ptr(X), dtype, Mc, K, N, group, int(bool(sym)),
                                  _ptr(alphas), alphas.shape[0], _ptr(err), _ptr(s_all),
                                  ctypes.byref(best))
    if st != OK:
        raise OracleError(f"w4ref_awq_search status {st}")
    return err, s_all, int(best.value)


def round_e4m3(v: float) -> float:
    """Nearest E4M3 value to v (ties to even), saturating at +-448."""
    return float(_load().w4ref_round_e4m3(float(v)))


def e4m3_to_f64(c: int) -> float:
    return float(_load().w4ref_e4m3_to_f64(int(c)))


def smooth_scales(X, W, dtype: int, alpha: float = 0.5) -> np.ndarray:
    """SmoothQuant factors s [K] fp32 from calibration X [Mc][K] and W [N][K]."""
    X = _bits16(X)
    W = _bits16(W)
    Mc, K = X.shape
    N = W.shape[0]
    s = np.zeros(K, np.float32)
    st = _load().w4ref_smooth_scales(_ptr(X), _ptr(W), dtype, Mc, K, N, float(alpha), _ptr(s))
    if st != OK:
        raise OracleError(f"w4ref_smooth_scales status {st}")
    return s


def quant8(A, dtype: int, fmt: int, col=None, col_op: int = 0):
    """Per-tensor 8-bit quantization of A [rows][K] -> (q uint8 [rows][K], scale f32).
    col_op: 0 none, 1 multiply by col[k], 2 divide by col[k]."""
    A = _bits16(A)
    rows, K = A.shape
    if col is not None:
        col = np.ascontiguousarray(col, dtype=np.float32)
    q = np.zeros((rows, K), np.uint8)
    sc = np.zeros(1, np.float32)
    st = _load().w4ref_quant8(_ptr(A), dtype, rows, K, _ptr(col), int(col_op), int(fmt), _ptr(q),
                              _ptr(sc))
    if st != OK:
        raise OracleError(f"w4ref_quant8 status {st}")
    return q, np.float32(sc[0])


def gemm8(Xq, Wq, fmt: int, sx, sw, dtype: int, rows=None) -> np.ndarray:
    """W8A8 layer on quantized operands (see w4ref_gemm8): [M or len(rows)][N] fp64."""
    Xq = np.ascontiguousarray(Xq, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    M, K = Xq.shape
    N = Wq.shape[0]
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rows.shape[0]
    else:
        nr = M
    Y = np.zeros((nr, N), np.float64)
    st = _load().w4ref_gemm8(_ptr(Xq), _ptr(Wq), int(fmt), M, K, N, float(sx), float(sw), dtype,
                             _ptr(rows), nr, _ptr(Y))
    if st != OK:
        raise OracleError(f"w4ref_gemm8 status {st}")
    return Y


def gptq_hessian(X, dtype: int) -> np.ndarray:
    """H = 2 X^T X in fp64 ([K][K]) from calibration activations X [Mc][K]."""
    X = _bits16(X)
    Mc, K = X.shape
    H = np.zeros((K, K), np.float64)
    st = _load().w4ref_gptq_hessian(_ptr(X), dtype, Mc, K, _ptr(H))
    if st != OK:
        raise OracleError(f"w4ref_gptq_hessian status {st}")
    return H


def gptq_inverse_factor(H: np.ndarray, percdamp: float = 0.01) -> np.ndarray:
    """U (upper, fp64) with U^T U = (H + lambda I)^-1, lambda = percdamp * mean(diag H).

    Library steps (numpy.linalg): the inverse of the damped Hessian, then its
    Cholesky factor; U = L^T for the lower factor L."""
    H = np.array(H, dtype=np.float64, copy=True)
    lam = percdamp * float(np.mean(np.diag(H)))
    H[np.diag_indices_from(H)] += lam
    Hinv = np.linalg.inv(H)
    Hinv = (Hinv + Hinv.T) / 2
    return np.linalg.cholesky(Hinv).T.copy()


def gptq_quantize(W, dtype: int, U, group: int, sym: bool):
    """The GPTQ column loop over W [N][K] given the fp32 factor U [K][K];
    returns (packed, scales, zeros) in the w4_quantize layout."""
    W = _bits16(W)
    N, K = W.shape
    U = np.ascontiguousarray(U, dtype=np.float32)
    assert U.shape == (K, K)
    G = K // group
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, G), np.float32)
    zeros = np.zeros((N, G), np.float32)
    st = _load().w4ref_gptq_quantize(_ptr(W), dtype, K, N, group, int(bool(sym)), _ptr(U),
                                     _ptr(packed), _ptr(scales), _ptr(zeros))
    if st != OK:
        raise OracleError(f"w4ref_gptq_quantize status {st}")
    return packed, scales, zeros


def gptq(W, X, dtype: int, group: int, sym: bool, percdamp: float = 0.01):
    """Whole GPTQ for one layer: Hessian, damped inverse factor (rounded to
    fp32), column loop.  Returns (packed, scales, zeros, U32)."""
    U32 = gptq_inverse_factor(gptq_hessian(X, dtype), percdamp).astype(np.float32)
    return (*gptq_quantize(W, dtype, U32, group, sym), U32)
