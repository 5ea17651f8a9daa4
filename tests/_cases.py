"""Prepared layers for parity tests: seeded inputs + the oracle's offline prep.

Every input the CUDA path receives here comes from svdq_inputs (seeded
synthetic data) and the CPU oracle's preparation (smoothing factors, low-rank
factors, residual); every expected value comes from the oracle.
"""

from __future__ import annotations

import dataclasses
import functools
from typing import Optional

import numpy as np

import oracle
from svdq_inputs import make_layer_inputs


@dataclasses.dataclass
class Prepared:
    name: str
    M: int
    K: int
    N: int
    r: int
    X: np.ndarray                # uint16 bf16 bits [M][K]
    lam: np.ndarray              # fp32 [K]
    inv: np.ndarray              # fp32 [K]
    L1: Optional[np.ndarray]     # uint16 bf16 bits [K][r]
    L2: Optional[np.ndarray]     # uint16 bf16 bits [r][N]
    R: np.ndarray                # fp32 [K][N]
    bias: Optional[np.ndarray]   # uint16 bf16 bits [N]


@functools.lru_cache(maxsize=8)
def prepare(workload: str, M=None, K=None, N=None, r=None, cal_rows=None) -> Prepared:
    """The oracle's preparation of a workload.  A workload that carries a
    LoRA adapter gets it joined to the low-rank branch (the oracle's
    attach_lora), so that ``r`` is then the SVD rank plus the adapter's."""
    li = make_layer_inputs(workload, M=M, K=K, N=N, r=r, cal_rows=cal_rows)
    lam, inv = oracle.smooth(li.Xcal, li.W)
    L1, L2, R, _ = oracle.lowrank(li.W, lam, li.r)
    rank = li.r
    if li.r == 0:
        L1 = L2 = None
    if li.lora_A is not None:
        L1, L2 = oracle.attach_lora(L1, L2, lam, li.lora_A, li.lora_B)
        rank += li.lora_A.shape[1]
    return Prepared(li.name, li.M, li.K, li.N, rank, li.X, lam, inv, L1, L2, R, li.bias)


def to_device(p: Prepared):
    """Torch CUDA tensors of a prepared layer (bf16 via bit views)."""
    import torch

    def bf16(a):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    return dict(
        X=bf16(p.X),
        inv=torch.from_numpy(p.inv).cuda(),
        L1=bf16(p.L1),
        L2=bf16(p.L2),
        R=torch.from_numpy(p.R).cuda(),
        bias=bf16(p.bias),
    )


def bf16_to_np_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
