"""ctypes binding of libsvdq.so: argument marshalling only.

Torch is used for device memory and the current CUDA stream; the calls below
pass raw pointers and sizes to the C ABI (include/svdq.h) and raise
``SvdqError`` on any non-zero status.  Output tensors are allocated here with
torch when the caller does not pass them.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libsvdq.so")

_P = ctypes.c_void_p
_I64 = ctypes.c_int64

SVDQ_OK = 0
SVDQ_ERR_TIMEOUT = 5


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)} ({status})")


_lib: Optional[ctypes.CDLL] = None


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libsvdq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} is missing: build it with `python -m bit_w4a4_quantized_smooth_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        L.svdq_status_string.restype = ctypes.c_char_p
        L.svdq_status_string.argtypes = [ctypes.c_int]
        L.svdq_packed_sizes.restype = ctypes.c_int
        L.svdq_packed_sizes.argtypes = [_I64, _I64, ctypes.POINTER(ctypes.c_size_t),
                                        ctypes.POINTER(ctypes.c_size_t)]
        L.svdq_pack_residual.restype = ctypes.c_int
        L.svdq_pack_residual.argtypes = [_P, _I64, _I64, _P, _P, _P]
        L.svdq_quantize_act.restype = ctypes.c_int
        L.svdq_quantize_act.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P]
        L.svdq_linear.restype = ctypes.c_int
        L.svdq_linear.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P]
        L.svdq_sync_status.restype = ctypes.c_int
        L.svdq_sync_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int)]
        L.svdq_selftest_wait_timeout.restype = ctypes.c_int
        L.svdq_selftest_wait_timeout.argtypes = [ctypes.c_uint64, _P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return load().svdq_status_string(status).decode()


def _check(status: int, what: str):
    if status != SVDQ_OK:
        raise SvdqError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def packed_sizes(rows: int, K: int) -> Tuple[int, int]:
    c = ctypes.c_size_t()
    s = ctypes.c_size_t()
    _check(load().svdq_packed_sizes(rows, K, ctypes.byref(c), ctypes.byref(s)), "svdq_packed_sizes")
    return c.value, s.value


def pack_residual(R, r_codes=None, r_scales=None, stream=None):
    """R fp32 [K][N] (cuda) -> (r_codes uint8 [N][K/2], r_scales uint8 tiled)."""
    import torch
    K, N = R.shape
    cb, sb = packed_sizes(N, K)
    if r_codes is None:
        r_codes = torch.empty((N, K // 2), dtype=torch.uint8, device=R.device)
    if r_scales is None:
        r_scales = torch.empty(sb, dtype=torch.uint8, device=R.device)
    _check(load().svdq_pack_residual(_ptr(R), K, N, _ptr(r_codes), _ptr(r_scales), _stream(stream)),
           "svdq_pack_residual")
    return r_codes, r_scales


def quantize_act(X, inv_lambda, L1, x_codes=None, x_scales=None, T=None, stream=None):
    """X bf16 [M][K], inv_lambda fp32 [K], L1 bf16 [K][r] or None ->
    (x_codes uint8 [M][K/2], x_scales uint8 tiled, T bf16 [M][r] or None)."""
    import torch
    M, K = X.shape
    r = 0 if L1 is None else L1.shape[1]
    cb, sb = packed_sizes(M, K)
    if x_codes is None:
        x_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    if x_scales is None:
        x_scales = torch.empty(sb, dtype=torch.uint8, device=X.device)
    if T is None and r > 0:
        T = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    _check(load().svdq_quantize_act(_ptr(X), _ptr(inv_lambda), _ptr(L1), M, K, r, _ptr(x_codes),
                                    _ptr(x_scales), _ptr(T), _stream(stream)), "svdq_quantize_act")
    return x_codes, x_scales, T


def linear(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M: int, K: int, N: int,
           Y=None, stream=None):
    """Fused 4-bit linear -> Y bf16 [M][N]."""
    import torch
    r = 0 if L2 is None else L2.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device)
    _check(load().svdq_linear(_ptr(x_codes), _ptr(x_scales), _ptr(T), _ptr(r_codes), _ptr(r_scales),
                              _ptr(L2), _ptr(bias), M, K, N, r, _ptr(Y), _stream(stream)),
           "svdq_linear")
    return Y


def sync_status(stream=None) -> Tuple[int, int]:
    """(status, wait id) recorded by the kernels since the last call."""
    where = ctypes.c_int(0)
    st = load().svdq_sync_status(_stream(stream), ctypes.byref(where))
    return st, where.value


def selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(load().svdq_selftest_wait_timeout(timeout_ns, _stream(stream)), "svdq_selftest_wait_timeout")
