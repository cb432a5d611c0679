"""ctypes binding for libglmq.so: the C ABI declared in include/glmq.h.

Argument marshalling only: every step of quantization and of the dequantizing
linear layer runs in the library's CUDA kernels. PyTorch is used for device
memory and streams. There is no CPU fallback: if the library is missing or the
device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libglmq.so")

# glmq_status values (include/glmq.h)
OK = 0
ERR_NULL_POINTER = 1
ERR_BAD_BITS = 2
ERR_BAD_SHAPE = 3
ERR_MISALIGNED = 4
ERR_CUDA = 5
ERR_DEVICE = 6
ERR_UNSUPPORTED_DEVICE = 7

DECODE_MAX_M = 16
DECODE_AUTO_MAX_M = 16
MAX_K = 65536
NOALLOC_SCRATCH_FLOATS = 1 << 20
EPILOGUE_NONE = 0
EPILOGUE_GEGLU = 1

#: every symbol include/glmq.h declares, with (restype, argtypes)
_c_int64 = ctypes.c_int64
_vp = ctypes.c_void_p
SIGNATURES = {
    "glmq_abi_version": (ctypes.c_int, []),
    "glmq_packed_bytes": (ctypes.c_size_t, [_c_int64, _c_int64, ctypes.c_int]),
    "glmq_quantize": (ctypes.c_int, [_vp, _c_int64, _c_int64, ctypes.c_int, _vp, _vp, _vp]),
    "glmq_quantize_geglu": (ctypes.c_int, [_vp, _c_int64, _c_int64, ctypes.c_int, _vp, _vp, _vp]),
    "glmq_quantize_zp": (ctypes.c_int, [_vp, _c_int64, _c_int64, _vp, _vp, _vp, _vp]),
    "glmq_gemm_zp": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _vp, _c_int64, _c_int64, _vp, _vp]),
    "glmq_gemm_fused": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, ctypes.c_int,
                                       _vp, _vp]),
    "glmq_gemm": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, _vp, _vp]),
    "glmq_gemm_decode": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, _vp, _vp]),
    "glmq_gemm_prefill": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, _vp, _vp]),
    "glmq_gemm_decode_prefetch": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, _vp,
                                                 _vp, _c_int64, _c_int64, _c_int64, _vp]),
    "glmq_gemm_decode_noalloc": (ctypes.c_int, [_vp, _c_int64, _vp, _vp, _c_int64, _c_int64, ctypes.c_int, _vp,
                                                _vp]),
    "glmq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "glmq_last_cuda_error": (ctypes.c_int, []),
    "glmq_kernel_launches": (ctypes.c_uint64, []),
    "glmq_last_device_error": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "glmq_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
}

_lib = None
_lock = threading.Lock()


class GlmqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: glmq status {status} ({status_string(status)})"
        if status == ERR_CUDA:
            msg += f", cudaError {lib().glmq_last_cuda_error()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m int8_quantized_glmq_b200.build` "
                    "(there is no CPU fallback)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().glmq_status_string(int(status)).decode()


def abi_version() -> int:
    return lib().glmq_abi_version()


def packed_bytes(N: int, K: int, bits: int) -> int:
    return lib().glmq_packed_bytes(N, K, bits)


def _check(status: int, where: str) -> None:
    if status != OK:
        raise GlmqError(status, where)


# ----------------------------------------------------------------- raw-pointer calls
def raw_quantize(W: int, N: int, K: int, bits: int, packed: int, scale: int, stream: int = 0) -> int:
    return lib().glmq_quantize(W, N, K, bits, packed, scale, stream)


def raw_quantize_geglu(W: int, N: int, K: int, bits: int, packed: int, scale: int, stream: int = 0) -> int:
    return lib().glmq_quantize_geglu(W, N, K, bits, packed, scale, stream)


def raw_quantize_zp(W: int, N: int, K: int, packed: int, scale: int, zero: int, stream: int = 0) -> int:
    return lib().glmq_quantize_zp(W, N, K, packed, scale, zero, stream)


def raw_gemm_zp(X: int, M: int, packed: int, scale: int, zero: int, N: int, K: int, Y: int, stream: int = 0) -> int:
    return lib().glmq_gemm_zp(X, M, packed, scale, zero, N, K, Y, stream)


def raw_gemm_fused(X: int, M: int, packed: int, scale: int, bias: int, N: int, K: int, bits: int, epilogue: int,
                   Y: int, stream: int = 0) -> int:
    return lib().glmq_gemm_fused(X, M, packed, scale, bias, N, K, bits, epilogue, Y, stream)


def raw_gemm(X: int, M: int, packed: int, scale: int, N: int, K: int, bits: int, Y: int, stream: int = 0,
             route: str = "auto") -> int:
    fn = {"auto": lib().glmq_gemm, "decode": lib().glmq_gemm_decode, "prefill": lib().glmq_gemm_prefill,
          "decode_noalloc": lib().glmq_gemm_decode_noalloc}[route]
    return fn(X, M, packed, scale, N, K, bits, Y, stream)


def raw_gemm_decode_prefetch(X: int, M: int, packed: int, scale: int, N: int, K: int, bits: int, Y: int,
                             next_packed: int, next_M: int, next_N: int, next_K: int, stream: int = 0) -> int:
    return lib().glmq_gemm_decode_prefetch(X, M, packed, scale, N, K, bits, Y, next_packed, next_M, next_N, next_K,
                                           stream)


def kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded (graph replays not included)."""
    return int(lib().glmq_kernel_launches())


def last_device_error(stream: int = 0):
    """(status, flags): synchronizes the stream and reads/clears the device status word."""
    flags = ctypes.c_uint32(0)
    st = lib().glmq_last_device_error(stream, ctypes.byref(flags))
    return st, flags.value


def set_wait_limit_ns(limit_ns: int) -> None:
    """glmq_set_wait_limit_ns: the give-up limit of the kernels' pipeline waits on the current
    device (0 = the default 2 s). A test hook for the failure path; not for production."""
    _check(lib().glmq_set_wait_limit_ns(int(limit_ns)), "glmq_set_wait_limit_ns")


# ----------------------------------------------------------------- torch-tensor calls
def _torch():
    import torch  # noqa: WPS433 (plumbing only)
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _require(t, dtype, ndim, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


class _on_device:
    """Makes t's device current for the call (a no-op when it already is)."""

    def __init__(self, t):
        torch = _torch()
        idx = t.device.index
        self._ctx = None if idx is None or idx == torch.cuda.current_device() else torch.cuda.device(idx)

    def __enter__(self):
        if self._ctx is not None:
            self._ctx.__enter__()

    def __exit__(self, *exc):
        if self._ctx is not None:
            self._ctx.__exit__(*exc)
        return False


def quantize(W, bits: int = 4, stream=None, out=None, geglu: bool = False):
    """One-shot quantization of fp16 W[N, K] -> (packed uint8 [N, K*bits/8], scale fp16 [N]).

    geglu=True stores the rows in the layout of the fused GeGLU epilogue
    (glmq_quantize_geglu); N must then be a multiple of 16."""
    torch = _torch()
    _require(W, torch.float16, 2, "W")
    N, K = W.shape
    if out is None:
        packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=W.device)
        scale = torch.empty((N,), dtype=torch.float16, device=W.device)
    else:
        packed, scale = out
    fn = raw_quantize_geglu if geglu else raw_quantize
    with _on_device(W):
        st = fn(W.data_ptr(), N, K, bits, packed.data_ptr(), scale.data_ptr(), _stream_ptr(stream))
    _check(st, "glmq_quantize_geglu" if geglu else "glmq_quantize")
    return packed, scale


def gemm(X, packed, scale, bits: int = 4, stream=None, out=None, route: str = "auto"):
    """Y[M, N] = fp16(s[n] * sum_k X[m,k] q[n,k]) for packed weights from :func:`quantize`."""
    torch = _torch()
    _require(X, torch.float16, 2, "X")
    _require(packed, torch.uint8, 2, "packed")
    _require(scale, torch.float16, 1, "scale")
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 8 != K * bits or scale.shape[0] != N:
        raise ValueError("packed/scale shapes do not match X and bits")
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if out is None else out
    with _on_device(X):
        st = raw_gemm(X.data_ptr(), M, packed.data_ptr(), scale.data_ptr(), N, K, bits, Y.data_ptr(),
                      _stream_ptr(stream), route)
    _check(st, f"glmq_gemm({route})")
    return Y


def gemm_fused(X, packed, scale, bits: int = 4, bias=None, epilogue: str = "none", stream=None, out=None):
    """glmq_gemm_fused: Y = fp16(s * X q + bias) [M, N], or with epilogue="geglu" (packed
    from quantize(..., geglu=True)) Y[m, j] = fp16(GELU(U[m, j]) * U[m, N/2 + j]) [M, N/2]."""
    torch = _torch()
    _require(X, torch.float16, 2, "X")
    _require(packed, torch.uint8, 2, "packed")
    _require(scale, torch.float16, 1, "scale")
    epi = {"none": EPILOGUE_NONE, "geglu": EPILOGUE_GEGLU}[epilogue]
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 8 != K * bits or scale.shape[0] != N:
        raise ValueError("packed/scale shapes do not match X and bits")
    if bias is not None:
        _require(bias, torch.float16, 1, "bias")
        if bias.shape[0] != N:
            raise ValueError("bias must have N entries")
    width = N // 2 if epi == EPILOGUE_GEGLU else N
    Y = torch.empty((M, width), dtype=torch.float16, device=X.device) if out is None else out
    with _on_device(X):
        st = raw_gemm_fused(X.data_ptr(), M, packed.data_ptr(), scale.data_ptr(),
                            0 if bias is None else bias.data_ptr(), N, K, bits, epi, Y.data_ptr(), _stream_ptr(stream))
    _check(st, "glmq_gemm_fused")
    return Y


def quantize_zp(W, stream=None, out=None):
    """Zero-point INT4 quantization of fp16 W[N, K] -> (packed uint8 [N, K/2], scale fp16 [N], zero uint8 [N])."""
    torch = _torch()
    _require(W, torch.float16, 2, "W")
    N, K = W.shape
    if out is None:
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
        scale = torch.empty((N,), dtype=torch.float16, device=W.device)
        zero = torch.empty((N,), dtype=torch.uint8, device=W.device)
    else:
        packed, scale, zero = out
    with _on_device(W):
        st = raw_quantize_zp(W.data_ptr(), N, K, packed.data_ptr(), scale.data_ptr(), zero.data_ptr(),
                             _stream_ptr(stream))
    _check(st, "glmq_quantize_zp")
    return packed, scale, zero


def gemm_zp(X, packed, scale, zero, stream=None, out=None):
    """Y[M, N] = fp16(s[n] * sum_k X (q - z[n])) for codes from :func:`quantize_zp`."""
    torch = _torch()
    _require(X, torch.float16, 2, "X")
    _require(packed, torch.uint8, 2, "packed")
    _require(scale, torch.float16, 1, "scale")
    _require(zero, torch.uint8, 1, "zero")
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or scale.shape[0] != N or zero.shape[0] != N:
        raise ValueError("packed/scale/zero shapes do not match X")
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if out is None else out
    with _on_device(X):
        st = raw_gemm_zp(X.data_ptr(), M, packed.data_ptr(), scale.data_ptr(), zero.data_ptr(), N, K, Y.data_ptr(),
                         _stream_ptr(stream))
    _check(st, "glmq_gemm_zp")
    return Y


def gemm_decode(X, packed, scale, bits: int = 4, stream=None, out=None):
    return gemm(X, packed, scale, bits, stream, out, route="decode")


def gemm_decode_prefetch(X, packed, scale, bits: int = 4, next_packed=None, next_M: int = 1, stream=None, out=None):
    """glmq_gemm_decode_prefetch: the decode GEMM (M <= 16), which also prefetches into L2
    the first weight tiles of the next decode call (``next_packed``, same bits, called
    with ``next_M`` tokens). Y is computed exactly as by :func:`gemm_decode`."""
    torch = _torch()
    _require(X, torch.float16, 2, "X")
    _require(packed, torch.uint8, 2, "packed")
    _require(scale, torch.float16, 1, "scale")
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 8 != K * bits or scale.shape[0] != N:
        raise ValueError("packed/scale shapes do not match X and bits")
    nptr, nN, nK = 0, 0, 0
    if next_packed is not None:
        _require(next_packed, torch.uint8, 2, "next_packed")
        nptr, nN, nK = next_packed.data_ptr(), next_packed.shape[0], next_packed.shape[1] * 8 // bits
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if out is None else out
    with _on_device(X):
        st = raw_gemm_decode_prefetch(X.data_ptr(), M, packed.data_ptr(), scale.data_ptr(), N, K, bits, Y.data_ptr(),
                                      nptr, next_M, nN, nK, _stream_ptr(stream))
    _check(st, "glmq_gemm_decode_prefetch")
    return Y


def gemm_prefill(X, packed, scale, bits: int = 4, stream=None, out=None):
    return gemm(X, packed, scale, bits, stream, out, route="prefill")
