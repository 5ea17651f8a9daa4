"""Counter-based random numbers (SplitMix64 + Box-Muller) and bf16 rounding.

SplitMix64 is Steele, Lea and Flood's generator ("Fast splittable
pseudorandom number generators", OOPSLA 2014); its finaliser is the mixing
function applied here to a Weyl sequence.  Everything is vectorised numpy on
uint64 (wrap-around arithmetic) so that full FLUX-sized layers draw in seconds.
"""

from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on an array of uint64 (modifies a copy)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def stream_seed(seed: int, stream: int) -> int:
    """Derive an independent 64-bit stream seed from (seed, stream id)."""
    z = _mix(np.array([(seed * 0x100000001B3 + stream * 0x9E3779B97F4A7C15) & (2**64 - 1)],
                      dtype=np.uint64))
    return int(z[0])


class SplitMix64Stream:
    """Counter-based SplitMix64: word i = mix(seed + (i+1)*golden).

    ``take(n)`` returns the next n words and advances the counter, so draws
    are reproducible regardless of how a tensor is split into calls.
    """

    def __init__(self, seed: int):
        self.seed = np.uint64(seed & (2**64 - 1))
        self.counter = 0

    def take(self, n: int) -> np.ndarray:
        idx = np.arange(self.counter + 1, self.counter + 1 + n, dtype=np.uint64)
        self.counter += n
        with np.errstate(over="ignore"):
            z = self.seed + idx * _GOLDEN
        return _mix(z)


def uniform(stream: SplitMix64Stream, n: int) -> np.ndarray:
    """n uniforms in [0, 1) from the top 53 bits of each word (fp64)."""
    w = stream.take(n)
    return (w >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(stream: SplitMix64Stream, n: int) -> np.ndarray:
    """n standard normals (fp64) by Box-Muller on consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform(stream, 2 * m)
    u1 = u[0::2]
    u2 = u[1::2]
    rad = np.sqrt(-2.0 * np.log1p(-u1))  # 1-u1 in (0, 1]
    ang = 2.0 * np.pi * u2
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    return out[:n]


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values once, to nearest-even, to bf16; return uint16 bits.

    Valid for finite values whose magnitude lies in bf16's normal range or
    is zero (all generated data): rounding is done on the fp64 bit pattern at
    the 8th significant bit, the result is exactly representable in fp32 and
    its top 16 bits are the bf16 pattern.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = x.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    with np.errstate(over="ignore"):
        r = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)
