"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

A thin ctypes wrapper around ``svdq_oracle.cpp`` (plain C++17 + OpenMP, fp64
where the contract allows).  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library never loads it, and it shares no code with the CUDA path.

Parity status of each function (what pins it, see ``tests/test_oracle_*.py``):

* codecs (bf16, E4M3, E2M1): exhaustive tables, hand-listed ties and
  special values, cross-checks against torch's own fp8/bf16 casts;
* group quantiser: error bound, scale bound, worked hand examples;
* layouts (code nibbles, 128x4 scale tiles): bijection, round trip and
  hand-computed offsets;
* smoothing: closed-form max-equalisation and the X W identity;
* eigen/SVD: numpy.linalg.svd / eigh on small inputs, Eckart-Young-Mirsky,
  exact reconstruction;
* quantised forward: brute-force quadruple loops on tiny inputs.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svdq_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (g++, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", _LIB + ".tmp", _SRC]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_from_f64.restype = ctypes.c_uint16
        L.oracle_bf16_from_f64.argtypes = [ctypes.c_double]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_nvfp4_quantize_group.restype = None
        L.oracle_nvfp4_quantize_group.argtypes = [_P, _P, _P]
        L.oracle_scale_offset.restype = _I64
        L.oracle_scale_offset.argtypes = [_I64, _I64, _I64]
        L.oracle_scale_bytes.restype = _I64
        L.oracle_scale_bytes.argtypes = [_I64, _I64]
        for name, args in [
            ("oracle_quantize_rows", [_P, _I64, _I64, _P, _P]),
            ("oracle_pack_residual", [_P, _I64, _I64, _P, _P]),
            ("oracle_smooth", [_P, _I64, _P, _I64, _I64, _P, _P]),
            ("oracle_sym_eig_top", [_P, _I64, _I64, _P, _P]),
            ("oracle_svd_top", [_P, _I64, _I64, _I64, _P, _P, _P]),
            ("oracle_lowrank", [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P]),
            ("oracle_attach_lora", [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P]),
            ("oracle_quantize_act", [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P]),
            ("oracle_dequant", [_P, _P, _I64, _I64, _P]),
            ("oracle_linear_rows", [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _I64, _P]),
            ("oracle_quantize_group_gs", [_P, ctypes.c_float, _P, _P]),
            ("oracle_quantize_act_ex", [_P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_float, _P, _P, _P]),
            ("oracle_quantize_rows_gs", [_P, _I64, _I64, ctypes.c_float, _P, _P]),
            ("oracle_pack_residual_gs", [_P, _I64, _I64, ctypes.c_float, _P, _P]),
            ("oracle_quantize_act_gs", [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P]),
            ("oracle_linear_rows_gs", [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_double,
                                       ctypes.c_double, _P, _I64, _P]),
        ]:
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = args
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_gelu.restype = ctypes.c_float
        L.oracle_gelu.argtypes = [ctypes.c_float]
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


# --------------------------------------------------------------- scalars ----

def bf16_to_f32(b: int) -> float:
    return lib().oracle_bf16_to_f32(b)


def bf16_from_f64(x: float) -> int:
    return lib().oracle_bf16_from_f64(x)


def e4m3_decode(c: int) -> float:
    return lib().oracle_e4m3_decode(c)


def e4m3_encode(x: float) -> int:
    return lib().oracle_e4m3_encode(x)


def e2m1_decode(c: int) -> float:
    return lib().oracle_e2m1_decode(c)


def e2m1_encode(x: float) -> int:
    return lib().oracle_e2m1_encode(x)


def quantize_group(v) -> tuple[np.ndarray, int]:
    v = np.ascontiguousarray(v, dtype=np.float32)
    assert v.shape == (16,)
    codes = np.zeros(16, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint8)
    lib().oracle_nvfp4_quantize_group(_ptr(v), _ptr(codes), _ptr(s))
    return codes, int(s[0])


def quantize_group_gs(v, g: float) -> tuple[np.ndarray, int]:
    """One group of 16 with the two-level quantiser (global scale g > 0)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    assert v.shape == (16,)
    codes = np.zeros(16, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint8)
    _check(lib().oracle_quantize_group_gs(_ptr(v), float(g), _ptr(codes), _ptr(s)), "quantize_group_gs")
    return codes, int(s[0])


def scale_offset(row: int, g: int, K: int) -> int:
    return lib().oracle_scale_offset(row, g, K)


def scale_bytes(rows: int, K: int) -> int:
    return lib().oracle_scale_bytes(rows, K)


def num_threads() -> int:
    return lib().oracle_num_threads()


# ---------------------------------------------------------------- arrays ----

def quantize_rows(V: np.ndarray):
    """fp32 [rows][K] -> (codes [rows][K/2] uint8, scales tiled uint8)."""
    V = np.ascontiguousarray(V, dtype=np.float32)
    rows, K = V.shape
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(rows, K), dtype=np.uint8)
    _check(lib().oracle_quantize_rows(_ptr(V), rows, K, _ptr(codes), _ptr(scales)), "quantize_rows")
    return codes, scales


def quantize_rows_gs(V: np.ndarray, g: float):
    """fp32 [rows][K] with global scale g -> (codes, scales)."""
    V = np.ascontiguousarray(V, dtype=np.float32)
    rows, K = V.shape
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(rows, K), dtype=np.uint8)
    _check(lib().oracle_quantize_rows_gs(_ptr(V), rows, K, float(g), _ptr(codes), _ptr(scales)),
           "quantize_rows_gs")
    return codes, scales


def pack_residual_gs(R: np.ndarray, gw: float):
    """R fp32 [K][N] with global scale g_w -> (r_codes [N][K/2], r_scales)."""
    R = np.ascontiguousarray(R, dtype=np.float32)
    K, N = R.shape
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(N, K), dtype=np.uint8)
    _check(lib().oracle_pack_residual_gs(_ptr(R), K, N, float(gw), _ptr(codes), _ptr(scales)),
           "pack_residual_gs")
    return codes, scales


def pack_residual(R: np.ndarray):
    """R fp32 [K][N] -> (r_codes [N][K/2], r_scales tiled over N rows)."""
    R = np.ascontiguousarray(R, dtype=np.float32)
    K, N = R.shape
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(N, K), dtype=np.uint8)
    _check(lib().oracle_pack_residual(_ptr(R), K, N, _ptr(codes), _ptr(scales)), "pack_residual")
    return codes, scales


def smooth(Xcal: np.ndarray, W: np.ndarray):
    """Smoothing factors (alpha = 0.5) -> (lambda fp32 [K], inv_lambda fp32 [K])."""
    Xcal = np.ascontiguousarray(Xcal, dtype=np.uint16)
    W = np.ascontiguousarray(W, dtype=np.uint16)
    Mc, K = Xcal.shape
    K2, N = W.shape
    assert K == K2
    lam = np.zeros(K, dtype=np.float32)
    inv = np.zeros(K, dtype=np.float32)
    _check(lib().oracle_smooth(_ptr(Xcal), Mc, _ptr(W), K, N, _ptr(lam), _ptr(inv)), "smooth")
    return lam, inv


def sym_eig_top(A: np.ndarray, k: int):
    A = np.ascontiguousarray(A, dtype=np.float64)
    n = A.shape[0]
    vals = np.zeros(k, dtype=np.float64)
    vecs = np.zeros((n, k), dtype=np.float64)
    _check(lib().oracle_sym_eig_top(_ptr(A), n, k, _ptr(vals), _ptr(vecs)), "sym_eig_top")
    return vals, vecs


def svd_top(A: np.ndarray, r: int):
    """Rank-r truncated SVD: (U [K][r], sigma [r+1], V [N][r])."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    K, N = A.shape
    U = np.zeros((K, r), dtype=np.float64)
    V = np.zeros((N, r), dtype=np.float64)
    s = np.zeros(r + 1, dtype=np.float64)
    _check(lib().oracle_svd_top(_ptr(A), K, N, r, _ptr(U), _ptr(s), _ptr(V)), "svd_top")
    return U, s, V


def lowrank(W: np.ndarray, lam: np.ndarray, r: int):
    """Offline prep -> (L1 bf16 bits [K][r], L2 bf16 bits [r][N], R fp32 [K][N], sigma [r+1])."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    K, N = W.shape
    L1 = np.zeros((K, r), dtype=np.uint16)
    L2 = np.zeros((r, N), dtype=np.uint16)
    R = np.zeros((K, N), dtype=np.float32)
    s = np.zeros(r + 1, dtype=np.float64)
    _check(lib().oracle_lowrank(_ptr(W), _ptr(lam), K, N, r, _ptr(L1), _ptr(L2), _ptr(R), _ptr(s)),
           "lowrank")
    return L1, L2, R, s


def attach_lora(L1: Optional[np.ndarray], L2: Optional[np.ndarray], lam: np.ndarray, A: np.ndarray,
                B: np.ndarray):
    """LoRA A [K][ra], B [ra][N] (bf16 bits) joined to the low-rank branch:
    -> (L1' [K][r+ra], L2' [r+ra][N]) bf16 bits; the residual is unchanged."""
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    K, ra = A.shape
    N = B.shape[1]
    r = 0 if L1 is None else L1.shape[1]
    L1c = np.zeros((K, 0), np.uint16) if L1 is None else np.ascontiguousarray(L1, dtype=np.uint16)
    L2c = np.zeros((0, N), np.uint16) if L2 is None else np.ascontiguousarray(L2, dtype=np.uint16)
    L1o = np.zeros((K, r + ra), dtype=np.uint16)
    L2o = np.zeros((r + ra, N), dtype=np.uint16)
    _check(lib().oracle_attach_lora(_ptr(L1c), _ptr(L2c), _ptr(lam), _ptr(A), _ptr(B), K, N, r, ra,
                                    _ptr(L1o), _ptr(L2o)), "attach_lora")
    return L1o, L2o


def quantize_act(X: np.ndarray, inv_lambda: np.ndarray, L1: Optional[np.ndarray], r: int):
    """-> (x_codes [M][K/2], x_scales tiled, T bf16 bits [M][r] or None)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    inv_lambda = np.ascontiguousarray(inv_lambda, dtype=np.float32)
    M, K = X.shape
    codes = np.zeros((M, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(M, K), dtype=np.uint8)
    T = np.zeros((M, r), dtype=np.uint16) if r > 0 else None
    L1c = None if r == 0 else np.ascontiguousarray(L1, dtype=np.uint16)
    _check(lib().oracle_quantize_act(_ptr(X), _ptr(inv_lambda), _ptr(L1c), M, K, r, _ptr(codes),
                                     _ptr(scales), _ptr(T)), "quantize_act")
    return codes, scales, T


def quantize_act_gs(X: np.ndarray, inv_lambda: np.ndarray, L1: Optional[np.ndarray], r: int, gx: float):
    """The activation step with global scale g_x for Xh (T is of Xh itself)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    inv_lambda = np.ascontiguousarray(inv_lambda, dtype=np.float32)
    M, K = X.shape
    codes = np.zeros((M, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(M, K), dtype=np.uint8)
    T = np.zeros((M, r), dtype=np.uint16) if r > 0 else None
    L1c = None if r == 0 else np.ascontiguousarray(L1, dtype=np.uint16)
    _check(lib().oracle_quantize_act_gs(_ptr(X), _ptr(inv_lambda), _ptr(L1c), M, K, r, float(gx), _ptr(codes),
                                        _ptr(scales), _ptr(T)), "quantize_act_gs")
    return codes, scales, T


def gelu(x: float) -> float:
    """GELU by Abramowitz and Stegun 7.1.28 in fp32 (the fused activation's rule)."""
    return lib().oracle_gelu(x)


def quantize_act_gelu(X: np.ndarray, inv_lambda: np.ndarray, L1: Optional[np.ndarray], r: int, gx: float = 0.0):
    """The activation step on GELU(X): Xh = RN_f32(GELU(x) * inv_lambda)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    inv_lambda = np.ascontiguousarray(inv_lambda, dtype=np.float32)
    M, K = X.shape
    codes = np.zeros((M, K // 2), dtype=np.uint8)
    scales = np.zeros(scale_bytes(M, K), dtype=np.uint8)
    T = np.zeros((M, r), dtype=np.uint16) if r > 0 else None
    L1c = None if r == 0 else np.ascontiguousarray(L1, dtype=np.uint16)
    _check(lib().oracle_quantize_act_ex(_ptr(X), _ptr(inv_lambda), _ptr(L1c), M, K, r, 1, float(gx), _ptr(codes),
                                        _ptr(scales), _ptr(T)), "quantize_act_gelu")
    return codes, scales, T


def linear_rows_gs(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M, K, N, r, gx, gw, rows) -> np.ndarray:
    """fp64 output rows with global scales: g_x g_w sum deq deq + T L2 + bias."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.zeros((len(rows), N), dtype=np.float64)
    args = [np.ascontiguousarray(a) if a is not None else None
            for a in (x_codes, x_scales, T, r_codes, r_scales, L2, bias)]
    _check(lib().oracle_linear_rows_gs(*[_ptr(a) for a in args], M, K, N, r, float(gx), float(gw), _ptr(rows),
                                       len(rows), _ptr(Y)), "linear_rows_gs")
    return Y


def dequant(codes: np.ndarray, scales: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.zeros((rows, K), dtype=np.float32)
    _check(lib().oracle_dequant(_ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)),
                                rows, K, _ptr(out)), "dequant")
    return out


def linear_rows(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M, K, N, r, rows) -> np.ndarray:
    """fp64 output rows Y[rows][N] of the quantised layer."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.zeros((len(rows), N), dtype=np.float64)
    args = [np.ascontiguousarray(a) if a is not None else None
            for a in (x_codes, x_scales, T, r_codes, r_scales, L2, bias)]
    _check(lib().oracle_linear_rows(*[_ptr(a) for a in args], M, K, N, r, _ptr(rows), len(rows),
                                    _ptr(Y)), "linear_rows")
    return Y
