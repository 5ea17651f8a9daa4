"""Synthetic layer workloads: shapes and value distributions, no method arithmetic.

Distributions (std written as N(0, std)):

* activations, kind ``"outlier"``: X ~ N(0, 1) with a seeded set of input
  channels multiplied by a per-channel factor (the outliers that smoothing
  migrates into the weights);
* activations, kind ``"gelu"``: X = GELU(z), z ~ N(0, 1), exact erf form,
  the skewed non-negative-heavy input of an MLP down-projection;
* weights, kind ``"planted"``: W ~ N(0, 0.02) plus a planted rank-q term
  sum_i s_i u_i v_i^T with orthonormal u, v and s_i = 10 x 0.02 (sqrt K + sqrt N),
  i.e. ten times the top singular value of the Gaussian bulk;
* weights, kind ``"gauss"``: W ~ N(0, 0.02);
* bias: None, or N(0, std).

Every tensor is rounded once to bf16 and returned as uint16 bit patterns.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from .generator import SplitMix64Stream, bf16_bits_from_f64, normal, stream_seed, uniform

# Stream ids: one independent SplitMix64 stream per tensor role.
_S_X, _S_W, _S_BIAS, _S_CH, _S_CHF, _S_U, _S_V, _S_XCAL, _S_LORA_A, _S_LORA_B = range(10)


@dataclasses.dataclass
class LayerInputs:
    """Inputs of one SVDQuant linear: Y = X W + bias, X [M][K], W [K][N]."""

    name: str
    M: int
    K: int
    N: int
    r: int
    X: np.ndarray                 # uint16 bf16 bits [M][K]
    W: np.ndarray                 # uint16 bf16 bits [K][N]
    bias: Optional[np.ndarray]    # uint16 bf16 bits [N] or None
    Xcal: np.ndarray              # uint16 bf16 bits [Mc][K], calibration rows for smoothing
    lora_A: Optional[np.ndarray] = None  # uint16 bf16 bits [K][r_lora]
    lora_B: Optional[np.ndarray] = None  # uint16 bf16 bits [r_lora][N]


def _outlier_channels(seed: int, K: int, n_out: int, lo: float, hi: float):
    """Seeded distinct channel indices and their scale factors."""
    s = SplitMix64Stream(stream_seed(seed, _S_CH))
    order = np.argsort(uniform(s, K), kind="stable")
    ch = np.sort(order[:n_out])
    f = SplitMix64Stream(stream_seed(seed, _S_CHF))
    if lo == hi:
        fac = np.full(n_out, lo, dtype=np.float64)
    else:
        fac = lo + (hi - lo) * uniform(f, n_out)
    return ch, fac


def make_activation(seed: int, stream: int, M: int, K: int, kind: str,
                    n_out: int = 0, lo: float = 1.0, hi: float = 1.0) -> np.ndarray:
    """Activation rows [M][K] as bf16 bits.

    ``stream`` selects the row stream (calibration and per-M sweeps use
    different streams) while the outlier channel set depends on ``seed`` only,
    so every draw of one layer shares the same outlier channels.
    """
    z = normal(SplitMix64Stream(stream_seed(seed, stream)), M * K).reshape(M, K)
    if kind == "outlier":
        if n_out:
            ch, fac = _outlier_channels(seed, K, n_out, lo, hi)
            z[:, ch] *= fac[None, :]
    elif kind == "gelu":
        from scipy.special import erf
        z = 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return bf16_bits_from_f64(z)


def make_weight(seed: int, K: int, N: int, kind: str, planted_rank: int = 0,
                std: float = 0.02) -> np.ndarray:
    """Weight [K][N] as bf16 bits (Gaussian bulk, optional planted low rank)."""
    w = std * normal(SplitMix64Stream(stream_seed(seed, _S_W)), K * N).reshape(K, N)
    if kind == "planted" and planted_rank > 0:
        q = min(planted_rank, K, N)
        gu = normal(SplitMix64Stream(stream_seed(seed, _S_U)), K * q).reshape(K, q)
        gv = normal(SplitMix64Stream(stream_seed(seed, _S_V)), N * q).reshape(N, q)
        u, _ = np.linalg.qr(gu)
        v, _ = np.linalg.qr(gv)
        s = 10.0 * std * (np.sqrt(K) + np.sqrt(N))
        w += s * (u @ v.T)
    elif kind not in ("gauss", "planted"):
        raise ValueError(f"unknown weight kind {kind!r}")
    return bf16_bits_from_f64(w)


def make_bias(seed: int, N: int, std: Optional[float]) -> Optional[np.ndarray]:
    if std is None:
        return None
    return bf16_bits_from_f64(std * normal(SplitMix64Stream(stream_seed(seed, _S_BIAS)), N))


def make_lora(seed: int, K: int, N: int, r_lora: int, std: float = 0.01):
    a = std * normal(SplitMix64Stream(stream_seed(seed, _S_LORA_A)), K * r_lora).reshape(K, r_lora)
    b = std * normal(SplitMix64Stream(stream_seed(seed, _S_LORA_B)), r_lora * N).reshape(r_lora, N)
    return bf16_bits_from_f64(a), bf16_bits_from_f64(b)


# ---------------------------------------------------------------------------
# The five layer workloads.  Each entry fixes shapes and distributions; the
# seed is 0x5EED0000 + 1000 * config + layer index.
# ---------------------------------------------------------------------------

CONFIGS = {
    "tiny": dict(config=1, M=256, K=1024, N=1024, r=16, x="outlier", n_out=8, lo=50.0, hi=50.0,
                 w="planted", q=4, bias=None),
    "flux_qkv": dict(config=2, M=4608, K=3072, N=9216, r=32, x="outlier", n_out=31, lo=20.0,
                     hi=100.0, w="planted", q=8, bias=0.01),
    "flux_mlp_up": dict(config=3, M=4608, K=3072, N=12288, r=32, x="outlier", n_out=31, lo=20.0,
                        hi=100.0, w="gauss", q=0, bias=None),
    "flux_mlp_down": dict(config=3, layer=1, M=4608, K=12288, N=3072, r=32, x="gelu", n_out=0,
                          lo=1.0, hi=1.0, w="gauss", q=0, bias=None),
    "sweep_3072": dict(config=4, M=4608, K=3072, N=3072, r=32, x="outlier", n_out=31, lo=20.0,
                       hi=100.0, w="planted", q=8, bias=0.01),
    # the two shapes of the synthetic DiT stack that no other workload has
    # (a single-stream block's fused input and output projections), with the
    # stack's rank-32 LoRA adapter; seeds are those of stack layers 76 and 77
    "dit_single_in": dict(config=5, layer=76, M=4608, K=3072, N=21504, r=32, x="outlier", n_out=31,
                          lo=20.0, hi=100.0, w="gauss", q=0, bias=None, lora=32),
    "dit_single_out": dict(config=5, layer=77, M=4608, K=15360, N=3072, r=32, x="gelu", n_out=0,
                           lo=1.0, hi=1.0, w="gauss", q=0, bias=None, lora=32),
}

# LoRA adapter of every DiT-stack layer: rank 32, A ~ N(0, 0.01), B ~ N(0, 0.01)
STACK_LORA_RANK = 32

SWEEP_M = (1, 16, 64, 256, 1024, 4096, 16384)
SWEEP_R = (16, 32, 64, 128)


def config_seed(config: int, layer: int = 0) -> int:
    return 0x5EED0000 + 1000 * config + layer


def make_layer_inputs(name: str, M: Optional[int] = None, K: Optional[int] = None,
                      N: Optional[int] = None, r: Optional[int] = None,
                      seed: Optional[int] = None, cal_rows: Optional[int] = None,
                      x_stream: int = _S_X) -> LayerInputs:
    """Inputs for a named workload; shape overrides give scaled-down cases
    with the same distributions (used by the parity tests)."""
    c = dict(CONFIGS[name])
    M = c["M"] if M is None else M
    K = c["K"] if K is None else K
    N = c["N"] if N is None else N
    r = c["r"] if r is None else r
    if seed is None:
        seed = config_seed(c["config"], c.get("layer", 0))
    n_out = c["n_out"]
    if n_out and K != c["K"]:
        n_out = max(1, int(round(n_out * K / c["K"])))
    X = make_activation(seed, x_stream, M, K, c["x"], n_out, c["lo"], c["hi"])
    if cal_rows is None:
        Xcal = X
    else:
        Xcal = make_activation(seed, _S_XCAL, cal_rows, K, c["x"], n_out, c["lo"], c["hi"])
    W = make_weight(seed, K, N, c["w"], c["q"])
    bias = make_bias(seed, N, c["bias"])
    A = B = None
    if c.get("lora"):
        A, B = make_lora(seed, K, N, c["lora"])
    return LayerInputs(name=name, M=M, K=K, N=N, r=r, X=X, W=W, bias=bias, Xcal=Xcal,
                       lora_A=A, lora_B=B)


def make_stack_layer_inputs(layer: int, M: int = 4608, with_x: bool = True) -> LayerInputs:
    """Inputs of layer ``layer`` (0..151) of the synthetic 12B DiT stack:
    W ~ N(0, 0.02) [K][N], no bias, a rank-32 LoRA adapter, and (unless
    ``with_x`` is false) M activation rows, hidden-state-like (outlier
    channels) for the 3072-wide inputs and GELU for the MLP/fused outputs."""
    K, N, kind = stack_layer_shapes()[layer]
    seed = config_seed(5, layer)
    if with_x:
        n_out = 31 if kind == "outlier" else 0
        lo, hi = (20.0, 100.0) if kind == "outlier" else (1.0, 1.0)
        X = make_activation(seed, _S_X, M, K, kind, n_out, lo, hi)
    else:
        X = np.zeros((0, K), dtype=np.uint16)
    W = make_weight(seed, K, N, "gauss", 0)
    A, B = make_lora(seed, K, N, STACK_LORA_RANK)
    return LayerInputs(name=f"dit_stack[{layer}]", M=M, K=K, N=N, r=32, X=X, W=W, bias=None, Xcal=X,
                       lora_A=A, lora_B=B)


def stack_layer_shapes():
    """The 152 linears of the synthetic 12B DiT stack at hidden 3072.

    19 double-stream blocks x (QKV 3072->9216, out 3072->3072, MLP up
    3072->12288, MLP down 12288->3072) and 38 single-stream blocks x (fused
    3072->21504, fused out 15360->3072).  Returns (K, N, input kind) tuples.
    """
    shapes = []
    for _ in range(19):
        shapes += [(3072, 9216, "outlier"), (3072, 3072, "outlier"),
                   (3072, 12288, "outlier"), (12288, 3072, "gelu")]
    for _ in range(38):
        shapes += [(3072, 21504, "outlier"), (15360, 3072, "gelu")]
    return shapes
