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
        L.svdq_quantize_act.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.svdq_quantize_act_workspace.restype = ctypes.c_int
        L.svdq_quantize_act_workspace.argtypes = [_I64, _I64, _I64, ctypes.POINTER(ctypes.c_size_t)]
        L.svdq_linear.restype = ctypes.c_int
        L.svdq_linear.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P]
        L.svdq_sync_status.restype = ctypes.c_int
        L.svdq_sync_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int)]
        L.svdq_selftest_wait_timeout.restype = ctypes.c_int
        L.svdq_selftest_wait_timeout.argtypes = [ctypes.c_uint64, _P]
        L.svdq_set_wait_timeout.restype = ctypes.c_int
        L.svdq_set_wait_timeout.argtypes = [ctypes.c_uint64]
        L.svdq_quantize_act_noalloc.restype = ctypes.c_int
        L.svdq_quantize_act_noalloc.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P]
        L.svdq_attach_lora.restype = ctypes.c_int
        L.svdq_attach_lora.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P]
        L.svdq_set_linear_path.restype = ctypes.c_int
        L.svdq_set_linear_path.argtypes = [ctypes.c_int]
        L.svdq_set_launch_overlap.restype = ctypes.c_int
        L.svdq_set_launch_overlap.argtypes = [ctypes.c_int]
        L.svdq_quantize_act_gelu.restype = ctypes.c_int
        L.svdq_quantize_act_gelu.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.svdq_linear_scaled.restype = ctypes.c_int
        L.svdq_linear_scaled.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_float,
                                         _P, _P]
        L.svdq_channel_absmax.restype = ctypes.c_int
        L.svdq_channel_absmax.argtypes = [_P, _I64, _I64, _P, _P]
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


def quantize_act_workspace_bytes(M: int, K: int, r: int) -> int:
    n = ctypes.c_size_t()
    _check(load().svdq_quantize_act_workspace(M, K, r, ctypes.byref(n)), "svdq_quantize_act_workspace")
    return n.value


# Zero-filled scratch per (device, stream), grown on demand: the calls leave
# its counters at zero, and calls on one stream never overlap.
_workspaces = {}


def workspace(nbytes: int, device, stream=None):
    """A zero-initialised device buffer of at least `nbytes` bytes for calls
    on `stream` (the current stream by default)."""
    import torch
    if nbytes == 0:
        return None
    key = (str(device), _stream(stream))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def quantize_act(X, inv_lambda, L1, x_codes=None, x_scales=None, T=None, stream=None, workspace_buf=None,
                 gelu: bool = False):
    """X bf16 [M][K], inv_lambda fp32 [K], L1 bf16 [K][r] or None ->
    (x_codes uint8 [M][K/2], x_scales uint8 tiled, T bf16 [M][r] or None).
    The scratch the call needs comes from `workspace_buf` (zero-filled before
    its first use) or from the binding's per-stream buffer.  gelu=True runs
    svdq_quantize_act_gelu (GELU applied to X before smoothing)."""
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
    need = quantize_act_workspace_bytes(M, K, r)
    ws = workspace_buf if workspace_buf is not None else workspace(need, X.device, stream)
    fn = load().svdq_quantize_act_gelu if gelu else load().svdq_quantize_act
    _check(fn(_ptr(X), _ptr(inv_lambda), _ptr(L1), M, K, r, _ptr(x_codes), _ptr(x_scales), _ptr(T), _ptr(ws),
              0 if ws is None else ws.numel(), _stream(stream)),
           "svdq_quantize_act_gelu" if gelu else "svdq_quantize_act")
    return x_codes, x_scales, T


def linear(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M: int, K: int, N: int,
           Y=None, stream=None, alpha: float = 1.0):
    """Fused 4-bit linear -> Y bf16 [M][N]; `alpha` (a power of two) scales
    the accumulator before the bias (per-tensor global scales g_x g_w)."""
    import torch
    r = 0 if L2 is None else L2.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device)
    if alpha == 1.0:
        _check(load().svdq_linear(_ptr(x_codes), _ptr(x_scales), _ptr(T), _ptr(r_codes), _ptr(r_scales),
                                  _ptr(L2), _ptr(bias), M, K, N, r, _ptr(Y), _stream(stream)),
               "svdq_linear")
    else:
        _check(load().svdq_linear_scaled(_ptr(x_codes), _ptr(x_scales), _ptr(T), _ptr(r_codes), _ptr(r_scales),
                                         _ptr(L2), _ptr(bias), M, K, N, r, float(alpha), _ptr(Y),
                                         _stream(stream)), "svdq_linear_scaled")
    return Y


def quantize_act_noalloc(X, inv_lambda, L1, x_codes=None, x_scales=None, T=None, stream=None):
    """quantize_act with its scratch inside the library (svdq_quantize_act_noalloc):
    for callers that cannot allocate device memory or pass a workspace.  The
    outputs are allocated here only when not given."""
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
    _check(load().svdq_quantize_act_noalloc(_ptr(X), _ptr(inv_lambda), _ptr(L1), M, K, r, _ptr(x_codes),
                                            _ptr(x_scales), _ptr(T), _stream(stream)), "svdq_quantize_act_noalloc")
    return x_codes, x_scales, T


def attach_lora(L1, L2, lam, A, B, L1_out=None, L2_out=None, stream=None):
    """Join a LoRA adapter (A bf16 [K][ra], B bf16 [ra][N]) to the low-rank
    branch (L1 [K][r], L2 [r][N], or None for r = 0) on the device ->
    (L1' bf16 [K][r+ra], L2' bf16 [r+ra][N])."""
    import torch
    K, ra = A.shape
    N = B.shape[1]
    r = 0 if L1 is None else L1.shape[1]
    if L1_out is None:
        L1_out = torch.empty((K, r + ra), dtype=torch.bfloat16, device=A.device)
    if L2_out is None:
        L2_out = torch.empty((r + ra, N), dtype=torch.bfloat16, device=A.device)
    _check(load().svdq_attach_lora(_ptr(L1), _ptr(L2), _ptr(lam), _ptr(A), _ptr(B), K, N, r, ra, _ptr(L1_out),
                                   _ptr(L2_out), _stream(stream)), "svdq_attach_lora")
    return L1_out, L2_out


def channel_absmax(X, amax=None, stream=None):
    """Fold a bf16 [M][K] activation batch into the running per-channel
    max |X| (fp32 [K] on the device; zeros are allocated when `amax` is
    None).  Returns amax."""
    import torch
    M, K = X.shape
    if amax is None:
        amax = torch.zeros(K, dtype=torch.float32, device=X.device)
    _check(load().svdq_channel_absmax(_ptr(X), M, K, _ptr(amax), _stream(stream)), "svdq_channel_absmax")
    return amax


def sync_status(stream=None) -> Tuple[int, int]:
    """(status, wait id) recorded by the kernels since the last call."""
    where = ctypes.c_int(0)
    st = load().svdq_sync_status(_stream(stream), ctypes.byref(where))
    return st, where.value


def set_wait_timeout(timeout_ns: int):
    """Limit (ns) of every bounded wait in kernels launched from now on."""
    _check(load().svdq_set_wait_timeout(timeout_ns), "svdq_set_wait_timeout")


LINEAR_PATHS = {"auto": 0, "large": 1, "small": 2}


def set_linear_path(path: str):
    """Force svdq_linear's kernel: "auto" (by shape), "large" or "small"."""
    _check(load().svdq_set_linear_path(LINEAR_PATHS[path]), "svdq_set_linear_path")


def set_launch_overlap(enable: bool):
    """Whether the layer calls' kernels may start their set-up while the
    kernel ahead of them in the stream finishes (default True); results are
    the same either way."""
    _check(load().svdq_set_launch_overlap(1 if enable else 0), "svdq_set_launch_overlap")


def selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(load().svdq_selftest_wait_timeout(timeout_ns, _stream(stream)), "svdq_selftest_wait_timeout")
