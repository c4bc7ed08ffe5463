"""Python binding of libw4a16.so: per-group INT4 weight quantization and the
W4A16 linear layer on B200 (sm_100a).

Argument marshalling only.  Every computation runs in the CUDA kernels of
libw4a16.so; there is no Python or CPU fallback, and every call raises if the
library is missing or returns an error status.  PyTorch provides device
memory and streams.

The functions mirror the C ABI of include/w4a16.h, with tensors in place of
pointers:

    w4_quantize(W, group=128, sym=True, col_scale=None) -> (packed, scales, zeros)
    w4a16_workspace_bytes(M, K, N, group=128) -> int
    w4a16_gemm(X, packed, scales, zeros, group=128, out=None, workspace=None) -> Y
    w4_awq_search(W, Xcal, alphas, group=128, sym=False, quantize=False)
        -> (err, best_scale, best_index[, (packed, scales, zeros)])
    w4_gptq(W, Xcal, group=128, sym=False, percdamp=0.01) -> (packed, scales, zeros[, U])
    w4_gptq_quantize(W, U, group=128, sym=False) -> (packed, scales, zeros)
    w8_smooth_scales(X, W, alpha=0.5) -> s
    w8_quantize(A, fmt, col=None, col_op=W8_COL_NONE) -> (q, scale)
    w8_gemm(Xq, x_scale, Wq, w_scale, fmt, dtype) -> Y
    w8a8_linear(X, Wq, w_scale, fmt, s=None) -> Y
    w4_status_string(status) -> str
    w4_device_status(reset=True) -> int
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "W4Error", "load", "lib_path", "w4_quantize", "w4_quantize_into", "w4a16_workspace_bytes",
    "w4a16_gemm", "w4a16_gemm_into", "w4_status_string", "w4_device_status", "w4_abi_version",
    "w4_last_error", "w4a16_gemm_noalloc", "w4_selftest_wait_timeout", "w4_awq_search",
    "w4_awq_search_workspace_bytes", "w4_gptq", "w4_gptq_quantize", "w4_gptq_workspace_bytes",
    "w4_gptq_quantize_workspace_bytes", "w8_smooth_scales", "w8_quantize", "w8_gemm",
    "w8a8_workspace_bytes", "w8a8_linear", "W8_INT8", "W8_E4M3", "W8_COL_NONE", "W8_COL_MUL",
    "W8_COL_DIV",
    "Workspace", "W4_OK", "W4_ERR_INVALID_ARG", "W4_ERR_UNSUPPORTED", "W4_ERR_CUDA",
    "W4_ERR_TIMEOUT", "W4_ERR_BOUNDS", "W4_F16", "W4_BF16", "w4_debug_build",
    "w4_debug_first_failure",
]

W4_OK, W4_ERR_INVALID_ARG, W4_ERR_UNSUPPORTED, W4_ERR_CUDA, W4_ERR_TIMEOUT = 0, 1, 2, 3, 4
W4_ERR_BOUNDS = 5
W4_F16, W4_BF16 = 0, 1
W8_INT8, W8_E4M3 = 0, 1
W8_COL_NONE, W8_COL_MUL, W8_COL_DIV = 0, 1, 2

_PKG = os.path.dirname(os.path.abspath(__file__))
# W4_DEBUG=1 in the environment selects the build with in-kernel bounds checks
lib_path = os.path.join(_PKG, "lib", "libw4a16_debug.so" if os.environ.get("W4_DEBUG") == "1"
                        else "libw4a16.so")
_lib = None


class W4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = ""
        try:
            detail = load().w4_last_error().decode()
        except Exception:
            pass
        super().__init__(f"{fn} failed: {w4_status_string(status)} ({status}) {detail}".rstrip())


def load() -> ctypes.CDLL:
    """Load libw4a16.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(lib_path):
        raise RuntimeError(
            f"{lib_path} is missing: build it with `python -m weight_only_int4_pack_b200.build`")
    lib = ctypes.CDLL(lib_path)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.w4_quantize.argtypes = [P, I, I64, I64, I, I, P, P, P, P, P]
    lib.w4_quantize.restype = I
    lib.w4a16_workspace_bytes.argtypes = [I64, I64, I64, I]
    lib.w4a16_workspace_bytes.restype = SZ
    lib.w4a16_gemm.argtypes = [P, I, I64, P, P, P, I64, I64, I, P, P, SZ, P]
    lib.w4a16_gemm.restype = I
    lib.w4_device_status.argtypes = [I]
    lib.w4_device_status.restype = I
    lib.w4_status_string.argtypes = [I]
    lib.w4_status_string.restype = ctypes.c_char_p
    lib.w4_abi_version.argtypes = []
    lib.w4_abi_version.restype = I
    lib.w4a16_gemm_noalloc.argtypes = [P, I, I64, P, P, P, I64, I64, I, P, P]
    lib.w4a16_gemm_noalloc.restype = I
    lib.w4_selftest_wait_timeout.argtypes = [ctypes.c_uint, P]
    lib.w4_selftest_wait_timeout.restype = I
    lib.w4_debug_build.argtypes = []
    lib.w4_debug_build.restype = I
    lib.w4_debug_first_failure.argtypes = [ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.w4_debug_first_failure.restype = I
    lib.w4_awq_search_workspace_bytes.argtypes = [I64, I64, I64, I]
    lib.w4_awq_search_workspace_bytes.restype = SZ
    lib.w4_awq_search.argtypes = [P, P, I, I64, I64, I64, I, I, P, I, P, P, P, P, P, P, P, SZ, P]
    lib.w4_awq_search.restype = I
    F = ctypes.c_float
    lib.w4_gptq_workspace_bytes.argtypes = [I64, I64, I64, I]
    lib.w4_gptq_workspace_bytes.restype = SZ
    lib.w4_gptq_quantize_workspace_bytes.argtypes = [I64, I64, I]
    lib.w4_gptq_quantize_workspace_bytes.restype = SZ
    lib.w4_gptq.argtypes = [P, P, I, I64, I64, I64, I, I, F, P, P, P, P, P, SZ, P]
    lib.w4_gptq.restype = I
    lib.w4_gptq_quantize.argtypes = [P, I, I64, I64, I, I, P, P, P, P, P, SZ, P]
    lib.w4_gptq_quantize.restype = I
    lib.w8_smooth_scales.argtypes = [P, P, I, I64, I64, I64, F, P, P, SZ, P]
    lib.w8_smooth_scales.restype = I
    lib.w8_quantize.argtypes = [P, I, I64, I64, P, I, I, P, P, P]
    lib.w8_quantize.restype = I
    lib.w8_gemm.argtypes = [P, P, P, P, I, I64, I64, I64, P, I, P]
    lib.w8_gemm.restype = I
    lib.w8a8_workspace_bytes.argtypes = [I64, I64]
    lib.w8a8_workspace_bytes.restype = SZ
    lib.w8a8_linear.argtypes = [P, I, I64, I64, P, I, P, P, I64, P, P, SZ, P]
    lib.w8a8_linear.restype = I
    lib.w4_last_error.argtypes = []
    lib.w4_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return W4_F16
    if t.dtype == torch.bfloat16:
        return W4_BF16
    raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")


def _p(t):
    # ctypes turns a Python int into a void* argument (None into NULL)
    return None if t is None else t.data_ptr()


try:  # the raw handle of the current stream, without building a Stream object
    _raw_stream = torch._C._cuda_getCurrentRawStream
except AttributeError:  # pragma: no cover
    _raw_stream = None


def _stream(stream, device=None):
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device() if device is None else device)
    return torch.cuda.current_stream().cuda_stream


def _check_dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def w4_status_string(status: int) -> str:
    try:
        return load().w4_status_string(int(status)).decode()
    except RuntimeError:
        return str(status)


def w4_last_error() -> str:
    """Description of the last failure on this thread (which check or CUDA call)."""
    return load().w4_last_error().decode()


def w4_abi_version() -> int:
    return int(load().w4_abi_version())


# Bumped when a bounded wait is seen to have run out: a kernel that stopped
# partway may have left the arrival counters of a decode workspace armed, so
# every Workspace zero-fills itself again before its next use.
_ws_epoch = [0]


def w4_device_status(reset: bool = True) -> int:
    """Status word set by kernels whose bounded waits ran out, or whose
    W4_DEBUG bounds checks failed (synchronizes).  On W4_ERR_TIMEOUT or
    W4_ERR_BOUNDS every Workspace of this module is zero-filled again before
    its next use, as include/w4a16.h asks."""
    st = int(load().w4_device_status(int(bool(reset))))
    if st in (W4_ERR_TIMEOUT, W4_ERR_BOUNDS):
        _ws_epoch[0] += 1
    return st


def w4_debug_build() -> bool:
    """True if the loaded library was built with W4_DEBUG (in-kernel bounds checks)."""
    return bool(load().w4_debug_build())


def w4_debug_first_failure() -> tuple[int, int]:
    """(file id, source line) of the first failed W4_DEBUG check since the
    status word was last cleared; (0, 0) if none.  Synchronizes; does not clear."""
    f, ln = ctypes.c_int(0), ctypes.c_int(0)
    st = int(load().w4_debug_first_failure(ctypes.byref(f), ctypes.byref(ln)))
    if st != W4_OK:
        raise W4Error("w4_debug_first_failure", st)
    return f.value, ln.value


def w4_selftest_wait_timeout(timeout_us: int = 1000, stream=None) -> None:
    """Enqueue the failure-detection self-test: a kernel whose only wait can
    never complete times out after `timeout_us` and sets the device status
    word (read it with w4_device_status)."""
    st = load().w4_selftest_wait_timeout(int(timeout_us), _stream(stream))
    if st != W4_OK:
        raise W4Error("w4_selftest_wait_timeout", st)


def w4_quantize_into(W, packed, scales, zeros, group=128, sym=True, col_scale=None, stream=None):
    """Quantize W [N][K] into caller-provided packed [N][K/2] u8, scales/zeros [N][K/group] f32."""
    _check_dev(W, packed, scales, zeros, col_scale)
    N, K = W.shape
    st = load().w4_quantize(_p(W), _dt(W), K, N, int(group), int(bool(sym)), _p(col_scale),
                            _p(packed), _p(scales), _p(zeros), _stream(stream))
    if st != W4_OK:
        raise W4Error("w4_quantize", st)
    return packed, scales, zeros


def w4_quantize(W: torch.Tensor, group: int = 128, sym: bool = True, col_scale=None, stream=None):
    """Per-group INT4 RTN quantization of W [N][K] -> (packed, scales, zeros)."""
    N, K = W.shape
    G = K // group if group > 0 else 0
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, G), dtype=torch.float32, device=W.device)
    zeros = torch.empty((N, G), dtype=torch.float32, device=W.device)
    return w4_quantize_into(W, packed, scales, zeros, group, sym, col_scale, stream)


def w4a16_workspace_bytes(M: int, K: int, N: int, group: int = 128) -> int:
    return int(load().w4a16_workspace_bytes(int(M), int(K), int(N), int(group)))


class Workspace:
    """A zero-filled device workspace that grows on demand (one per stream).
    Zero-filled again after a bounded wait ran out (see w4_device_status)."""

    def __init__(self, device=None):
        self.buf = None
        self.device = device
        self.epoch = _ws_epoch[0]

    def get(self, nbytes: int, device):
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            self.epoch = _ws_epoch[0]
        elif self.epoch != _ws_epoch[0]:
            self.buf.zero_()
            self.epoch = _ws_epoch[0]
        return self.buf


_default_ws = {}


_ws_need = {}


def w4a16_gemm_into(X, packed, scales, zeros, Y, group=128, workspace=None, stream=None):
    """Y [M][N] = X [M][K] * dequant(packed, scales, zeros)^T into caller-provided Y."""
    _check_dev(X, packed, scales, zeros, Y)
    M, K = X.shape
    N = packed.shape[0]
    lib = _lib if _lib is not None else load()
    key = (M, K, N, group)
    need = _ws_need.get(key)
    if need is None:
        need = _ws_need[key] = int(lib.w4a16_workspace_bytes(M, K, N, int(group)))
    dev = X.device
    if isinstance(workspace, Workspace) or workspace is None:
        wsobj = workspace
        if wsobj is None:
            skey = (dev, _stream(stream, dev.index))
            wsobj = _default_ws.setdefault(skey, Workspace())
        ws = wsobj.get(need, dev)
    else:
        ws = workspace
    wsz = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib.w4a16_gemm(X.data_ptr(), _dt(X), M, packed.data_ptr(), scales.data_ptr(),
                        None if zeros is None else zeros.data_ptr(), K, N, group,
                        Y.data_ptr(), None if ws is None else ws.data_ptr(), wsz,
                        _stream(stream, dev.index))
    if st != W4_OK:
        raise W4Error("w4a16_gemm", st)
    return Y


def w4a16_gemm(X, packed, scales, zeros=None, group: int = 128, out=None, workspace=None,
               stream=None):
    """The W4A16 linear layer: Y = X * dequant(packed, scales, zeros)^T."""
    M = X.shape[0]
    N = packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=X.dtype, device=X.device)
    return w4a16_gemm_into(X, packed, scales, zeros, Y, group, workspace, stream)


def w4a16_gemm_noalloc(X, packed, scales, zeros=None, group: int = 128, out=None, stream=None):
    """The decode layer (M <= 32) with the library's own static scratch space:
    for callers that cannot allocate device memory.  Calls on one device must
    not overlap on the GPU (they share that scratch space)."""
    _check_dev(X, packed, scales, zeros, out)
    M, K = X.shape
    N = packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=X.dtype, device=X.device)
    st = load().w4a16_gemm_noalloc(_p(X), _dt(X), M, _p(packed), _p(scales), _p(zeros), K, N,
                                   int(group), _p(Y), _stream(stream))
    if st != W4_OK:
        raise W4Error("w4a16_gemm_noalloc", st)
    return Y


def w4_awq_search_workspace_bytes(Mc: int, K: int, N: int, group: int = 128) -> int:
    return int(load().w4_awq_search_workspace_bytes(int(Mc), int(K), int(N), int(group)))


def w4_awq_search(W, Xcal, alphas, group: int = 128, sym: bool = False, quantize: bool = False,
                  workspace=None, stream=None):
    """AWQ scale search: err[t] = ||Q(W*s_t)(Xcal/s_t) - Xcal W^T||_F^2 with
    s_t = (mean|Xcal| / mean|W|)^alphas[t] per input channel.

    Returns (err fp64 [n_alpha], best_scale fp32 [K], best_index int32 [1]),
    all on W's device, plus (packed, scales, zeros) = Q(W * best_scale) when
    quantize=True.  `workspace` is an optional uint8 device tensor of at
    least w4_awq_search_workspace_bytes bytes."""
    _check_dev(W, Xcal, workspace)
    N, K = W.shape
    Mc = Xcal.shape[0]
    if Xcal.dtype != W.dtype:
        raise TypeError("W and Xcal must share one dtype")
    a = [float(v) for v in alphas]
    al = (ctypes.c_float * len(a))(*a)
    lib = load()
    need = int(lib.w4_awq_search_workspace_bytes(Mc, K, N, int(group)))
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8,
                                                             device=W.device)
    dev = W.device
    err = torch.empty(len(a), dtype=torch.float64, device=dev)
    best_scale = torch.empty(K, dtype=torch.float32, device=dev)
    best_index = torch.empty(1, dtype=torch.int32, device=dev)
    q = None
    if quantize:
        G = K // group if group > 0 else 0
        q = (torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
             torch.empty((N, G), dtype=torch.float32, device=dev),
             torch.empty((N, G), dtype=torch.float32, device=dev))
    st = lib.w4_awq_search(_p(W), _p(Xcal), _dt(W), Mc, K, N, int(group), int(bool(sym)), al,
                           len(a), _p(err), _p(best_scale), _p(best_index),
                           *(_p(t) for t in (q or (None, None, None))), _p(ws),
                           ws.numel() * ws.element_size(), _stream(stream))
    if st != W4_OK:
        raise W4Error("w4_awq_search", st)
    if quantize:
        return err, best_scale, best_index, q
    return err, best_scale, best_index


# ---- GPTQ ------------------------------------------------------------------------------------

def w4_gptq_workspace_bytes(Mc: int, K: int, N: int, group: int = 128) -> int:
    return int(load().w4_gptq_workspace_bytes(int(Mc), int(K), int(N), int(group)))


def w4_gptq_quantize_workspace_bytes(K: int, N: int, group: int = 128) -> int:
    return int(load().w4_gptq_quantize_workspace_bytes(int(K), int(N), int(group)))


def _q_out(N, K, group, dev):
    G = K // group if group > 0 else 0
    return (torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
            torch.empty((N, G), dtype=torch.float32, device=dev),
            torch.empty((N, G), dtype=torch.float32, device=dev))


def w4_gptq(W, Xcal, group: int = 128, sym: bool = False, percdamp: float = 0.01,
            return_u: bool = False, workspace=None, stream=None):
    """GPTQ of W [N][K] with calibration activations Xcal [Mc][K] ->
    (packed, scales, zeros) in the w4_quantize layout (+ U [K][K] fp32 when
    return_u).  Synchronizes the stream once (factorization status)."""
    _check_dev(W, Xcal, workspace)
    N, K = W.shape
    Mc = Xcal.shape[0]
    if Xcal.dtype != W.dtype:
        raise TypeError("W and Xcal must share one dtype")
    p, s, z = _q_out(N, K, group, W.device)
    U = torch.empty((K, K), dtype=torch.float32, device=W.device) if return_u else None
    need = w4_gptq_workspace_bytes(Mc, K, N, group)
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8,
                                                             device=W.device)
    st = load().w4_gptq(_p(W), _p(Xcal), _dt(W), Mc, K, N, int(group), int(bool(sym)),
                        float(percdamp), _p(p), _p(s), _p(z), _p(U), _p(ws),
                        ws.numel() * ws.element_size(), _stream(stream))
    if st != W4_OK:
        raise W4Error("w4_gptq", st)
    return (p, s, z, U) if return_u else (p, s, z)


def w4_gptq_quantize(W, U, group: int = 128, sym: bool = False, workspace=None, stream=None):
    """The GPTQ column loop over W [N][K] given the fp32 factor U [K][K]."""
    _check_dev(W, U, workspace)
    N, K = W.shape
    p, s, z = _q_out(N, K, group, W.device)
    need = w4_gptq_quantize_workspace_bytes(K, N, group)
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8,
                                                             device=W.device)
    st = load().w4_gptq_quantize(_p(W), _dt(W), K, N, int(group), int(bool(sym)), _p(U), _p(p),
                                 _p(s), _p(z), _p(ws), ws.numel() * ws.element_size(),
                                 _stream(stream))
    if st != W4_OK:
        raise W4Error("w4_gptq_quantize", st)
    return p, s, z


# ---- W8A8 (SmoothQuant INT8 / FP8 E4M3) ---------------------------------------------------

def w8_smooth_scales(X, W, alpha: float = 0.5, stream=None):
    """SmoothQuant factors s [K] fp32 from calibration X [Mc][K] and W [N][K]."""
    _check_dev(X, W)
    Mc, K = X.shape
    N = W.shape[0]
    s = torch.empty(K, dtype=torch.float32, device=X.device)
    ws = torch.empty(8 * K, dtype=torch.uint8, device=X.device)
    st = load().w8_smooth_scales(_p(X), _p(W), _dt(X), Mc, K, N, float(alpha), _p(s), _p(ws),
                                 ws.numel(), _stream(stream))
    if st != W4_OK:
        raise W4Error("w8_smooth_scales", st)
    return s


def w8_quantize(A, fmt: int, col=None, col_op: int = W8_COL_NONE, stream=None):
    """Per-tensor 8-bit quantization of A [rows][K] -> (q uint8 [rows][K], scale f32 [2]
    holding (scale, amax))."""
    _check_dev(A, col)
    rows, K = A.shape
    q = torch.empty((rows, K), dtype=torch.uint8, device=A.device)
    scale = torch.empty(2, dtype=torch.float32, device=A.device)
    st = load().w8_quantize(_p(A), _dt(A), rows, K, _p(col), int(col_op), int(fmt), _p(q),
                            _p(scale), _stream(stream))
    if st != W4_OK:
        raise W4Error("w8_quantize", st)
    return q, scale


def w8_gemm(Xq, x_scale, Wq, w_scale, fmt: int, dtype=torch.float16, out=None, stream=None):
    """Y [M][N] = (Xq Wq^T) * x_scale[0] * w_scale[0] on 8-bit operands."""
    _check_dev(Xq, x_scale, Wq, w_scale, out)
    M, K = Xq.shape
    N = Wq.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=dtype, device=Xq.device)
    st = load().w8_gemm(_p(Xq), _p(x_scale), _p(Wq), _p(w_scale), int(fmt), M, K, N, _p(Y),
                        _dt(Y), _stream(stream))
    if st != W4_OK:
        raise W4Error("w8_gemm", st)
    return Y


def w8a8_workspace_bytes(M: int, K: int) -> int:
    return int(load().w8a8_workspace_bytes(int(M), int(K)))


def w8a8_linear(X, Wq, w_scale, fmt: int, s=None, out=None, workspace=None, stream=None):
    """The W8A8 layer: X [M][K] (16-bit) divided by s, quantized per tensor on
    the fly, times the quantized weights Wq [N][K]; Y [M][N] in X's dtype."""
    _check_dev(X, Wq, w_scale, s, out, workspace)
    M, K = X.shape
    N = Wq.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=X.dtype, device=X.device)
    need = w8a8_workspace_bytes(M, K)
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8,
                                                             device=X.device)
    st = load().w8a8_linear(_p(X), _dt(X), M, K, _p(s), int(fmt), _p(Wq), _p(w_scale), N, _p(Y),
                            _p(ws), ws.numel() * ws.element_size(), _stream(stream))
    if st != W4_OK:
        raise W4Error("w8a8_linear", st)
    return Y
