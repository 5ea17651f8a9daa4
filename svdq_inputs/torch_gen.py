"""The generator of ``generator.py`` on torch tensors, for any device.

Same definition: counter-based SplitMix64 words (Steele, Lea and Flood,
OOPSLA 2014), uniforms from their top 53 bits, Box-Muller normals, one
round-to-nearest-even to bf16 from fp64.  Unsigned 64-bit arithmetic is done
on int64 tensors (two's-complement wrap-around for + and *, logical right
shifts by masking).  Used where the CPU generator would take minutes: the
152 layers of the synthetic DiT stack (about 8e9 values) are drawn on the GPU.

The integer stream is bit-identical to the numpy one; the transcendental
steps (log1p, cos, sin, erf) may differ from numpy's by an ulp in fp64,
which changes the bf16 value in a tiny fraction of elements.
"""

from __future__ import annotations

import math

import numpy as np

from . import generator as _g
from .workloads import _S_LORA_A, _S_LORA_B, _S_W, _S_X, STACK_LORA_RANK, _outlier_channels, config_seed
from .workloads import stack_layer_shapes


def _s64(v: int) -> int:
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


_GOLDEN = _s64(int(_g._GOLDEN))
_M1 = _s64(int(_g._M1))
_M2 = _s64(int(_g._M2))


def _srl(z, k: int):
    """Logical right shift of int64 values holding uint64 bit patterns."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix(z):
    z = z ^ _srl(z, 30)
    z = z * _M1
    z = z ^ _srl(z, 27)
    z = z * _M2
    return z ^ _srl(z, 31)


def words(seed: int, counter0: int, n: int, device):
    """Words counter0 + 1 .. counter0 + n of the stream ``seed``."""
    import torch
    idx = torch.arange(counter0 + 1, counter0 + 1 + n, dtype=torch.int64, device=device)
    return _mix(_s64(seed) + idx * _GOLDEN)


def uniform(seed: int, n: int, device, counter0: int = 0):
    import torch
    return _srl(words(seed, counter0, n, device), 11).to(torch.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, n: int, device):
    """n standard normals (fp64), the same pairs as ``generator.normal``."""
    import torch
    m = (n + 1) // 2
    u = uniform(seed, 2 * m, device).view(m, 2)
    rad = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
    ang = (2.0 * math.pi) * u[:, 1]
    return torch.stack([rad * torch.cos(ang), rad * torch.sin(ang)], dim=1).reshape(-1)[:n]


def bf16_from_f64(x):
    """Round fp64 once, to nearest-even, to bf16 (finite normal or zero
    values), by the bit-pattern rule of ``generator.bf16_bits_from_f64``."""
    import torch
    u = x.contiguous().view(torch.int64)
    lsb = (u >> 45) & 1
    r = (u + ((1 << 44) - 1) + lsb) & ~((1 << 45) - 1)
    return r.view(torch.float64).to(torch.bfloat16)  # exact: 8 significant bits


def make_activation(seed: int, stream: int, M: int, K: int, kind: str, n_out: int, lo: float, hi: float,
                    device):
    import torch
    z = normal(_g.stream_seed(seed, stream), M * K, device).view(M, K)
    if kind == "outlier":
        if n_out:
            ch, fac = _outlier_channels(seed, K, n_out, lo, hi)
            z[:, torch.from_numpy(ch).to(device)] *= torch.from_numpy(fac).to(device)[None, :]
    elif kind == "gelu":
        z = 0.5 * z * (1.0 + torch.special.erf(z / math.sqrt(2.0)))
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return bf16_from_f64(z)


def make_weight_gauss(seed: int, K: int, N: int, device, std: float = 0.02):
    return bf16_from_f64(std * normal(_g.stream_seed(seed, _S_W), K * N, device).view(K, N))


def make_lora(seed: int, K: int, N: int, r_lora: int, device, std: float = 0.01):
    a = std * normal(_g.stream_seed(seed, _S_LORA_A), K * r_lora, device).view(K, r_lora)
    b = std * normal(_g.stream_seed(seed, _S_LORA_B), r_lora * N, device).view(r_lora, N)
    return bf16_from_f64(a), bf16_from_f64(b)


def make_stack_layer(layer: int, M: int, device, with_x: bool = True):
    """Layer ``layer`` of the synthetic DiT stack, as
    ``workloads.make_stack_layer_inputs`` defines it, drawn on ``device``:
    -> dict(X bf16 [M][K] (None without ``with_x``), W bf16 [K][N],
    A bf16 [K][32], B bf16 [32][N], K, N)."""
    K, N, kind = stack_layer_shapes()[layer]
    seed = config_seed(5, layer)
    n_out = 31 if kind == "outlier" else 0
    lo, hi = (20.0, 100.0) if kind == "outlier" else (1.0, 1.0)
    X = make_activation(seed, _S_X, M, K, kind, n_out, lo, hi, device) if with_x else None
    W = make_weight_gauss(seed, K, N, device)
    A, B = make_lora(seed, K, N, STACK_LORA_RANK, device)
    return dict(X=X, W=W, A=A, B=B, K=K, N=N)


__all__ = ["words", "uniform", "normal", "bf16_from_f64", "make_activation", "make_weight_gauss",
           "make_lora", "make_stack_layer"]
