"""Special values through the activation kernel itself (svdq_quantize_act).

The activation step decides zero groups, saturated and subnormal scales,
signed zeros and E2M1 rounding ties after the smoothing multiply.  Random
activations almost never reach those decisions, so this file builds X from
crafted 16-element groups and compares codes and scales byte for byte with
the oracle, and T within the parity tolerance.

Column bands use different smoothing reciprocals: 1, 1/2 and 2 (exact, so a
crafted Xh value survives the multiply) and 3/4 (the product is rounded to
fp32 first, as both sides do).  Each crafted group is written as X = Xh / inv
into a band whose reciprocal is a power of two.
"""

import numpy as np
import pytest

import oracle
from svdq_inputs import bf16_bits_from_f64
from tests._cases import bf16_to_np_bits

pytestmark = pytest.mark.gpu

K = 256            # four 64-column bands, 4 groups each
BAND_INV = (1.0, 0.5, 2.0, 0.75)
TIES = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _bf16_neighbours(x):
    """x and the bf16 values just below and above it."""
    b = int(bf16_bits_from_f64(np.array([x]))[0])
    out = []
    for d in (-1, 0, 1):
        v = ((b + d) & 0xFFFF) << 16
        out.append(float(np.array([v], dtype=np.uint32).view(np.float32)[0]))
    return out


def crafted_groups():
    """Groups of 16 smoothed values, each with a label (rounded once to bf16
    by build_case; the values a case turns on are bf16 numbers)."""
    g = []
    g.append(("zeros", [0.0] * 16))
    g.append(("negative zeros", [-0.0] * 16))
    g.append(("mixed zeros", [0.0, -0.0] * 8))
    # amax / 6 above 448: the scale saturates to 448, large codes to 6
    g.append(("saturated scale", [6144.0, -3072.0, 2688.0, 2700.0, -448.0, 1.0, 0.0, -0.0]
              + [1000.0 * i for i in range(8)]))
    g.append(("saturated, huge", [-32768.0, 16384.0, 4096.0] + [100.0] * 13))
    # subnormal E4M3 scales (2^-9 steps below 2^-6)
    for m in (1, 2, 3, 5, 7):
        a = 6.0 * m * 2.0 ** -9
        g.append((f"subnormal scale {m}", [a, -a / 2, a / 3, a / 4, a / 6, -a / 8, a / 12, 0.0]
                  + [a * i / 9 for i in range(8)]))
    # amax / 6 exactly half the smallest subnormal: the scale rounds to 0
    t = 6.0 * 2.0 ** -10
    g.append(("scale underflows to 0", [t, -t, t / 2, -t / 3] + [t / 5] * 12))
    # amax / 6 on an E4M3 rounding tie (1.0625 between 1.0 and 1.125)
    g.append(("scale tie", [6.375, -1.0, 0.5, 2.0] + [0.1 * i for i in range(12)]))
    g.append(("scale tie odd", [6.0 * 1.1875, 1.0, -2.0, 3.0] + [0.2 * i for i in range(12)]))
    # E2M1 ties with scale 1 (amax 6): every tie, its neighbours, both signs
    vals = []
    for x in TIES:
        vals += _bf16_neighbours(x)
    vals += [-v for v in vals]
    for i in range(0, len(vals), 15):
        chunk = vals[i:i + 15]
        chunk += [0.0] * (15 - len(chunk))
        g.append((f"e2m1 ties {i // 15}", [6.0] + chunk))
    # the same ties at scale 2 (amax 12): codes see v / 2
    g.append(("e2m1 ties at scale 2", [12.0] + [2.0 * x for x in TIES] + [-2.0 * x for x in TIES] + [0.0]))
    # values past 6 times the scale saturate to code magnitude 6
    g.append(("element saturation", [6.0, 6.0, -6.0, 5.99, 6.01] + [5.5, 5.0, 4.5] + [0.3] * 8))
    return g


def build_case(M=40, seed=7):
    """X bf16 bits [M][K] and inv_lambda [K]: crafted groups in the
    power-of-two bands, seeded normal values elsewhere."""
    rng = np.random.default_rng(seed)
    inv = np.repeat(np.array(BAND_INV, dtype=np.float32), 64)
    Xf = rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1)))
    groups = crafted_groups()
    slots = [(m, gi) for m in range(M) for gi in range(K // 16) if BAND_INV[gi // 4] != 0.75]
    assert len(groups) <= len(slots)
    exact = []
    for (label, vals), (m, gi) in zip(groups, slots):
        v = np.array(vals, dtype=np.float64)
        assert v.shape == (16,), label
        # each crafted value rounded once to bf16; the values a case is about
        # (zeros, ties, 6, the amax) are bf16 numbers already
        vb = (bf16_bits_from_f64(v).astype(np.uint32) << 16).view(np.float32)
        exact.append((label, vb))
        Xf[m, 16 * gi:16 * gi + 16] = vb.astype(np.float64) / inv[16 * gi]
    X = bf16_bits_from_f64(Xf)
    # X * inv reproduces the crafted group exactly (signed zeros included)
    for (label, vb), (m, gi) in zip(exact, slots):
        got = (X[m, 16 * gi:16 * gi + 16].astype(np.uint32) << 16).view(np.float32) * inv[16 * gi]
        assert np.array_equal(got.view(np.uint32), vb.view(np.uint32)), label
    return X, inv


def test_fixture_reaches_the_special_cases():
    """The oracle's own output shows every case the file is about: zero
    scales, the saturated scale 0x7E, subnormal scales, negative-zero codes."""
    X, inv = build_case()
    xc, xs, _ = oracle.quantize_act(X, inv, None, 0)
    assert 0 in xs                      # zero groups (and underflow)
    assert 0x7E in xs                   # 448
    assert any(0 < s < 8 for s in xs)   # subnormal E4M3
    nib = np.concatenate([xc & 15, xc >> 4])
    assert 8 in nib                     # -0 code
    assert 7 in nib and 15 in nib       # +6 and -6


@pytest.mark.parametrize("r", [0, 16, 32])
def test_quantize_act_special_values(r):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from tests.test_gpu_parity import check_T
    X, inv = build_case()
    M = X.shape[0]
    rng = np.random.default_rng(11)
    L1 = bf16_bits_from_f64(0.05 * rng.standard_normal((K, r))) if r else None
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    xc, xs, T = svdq.quantize_act(dev(X), torch.from_numpy(inv).cuda(), dev(L1) if r else None)
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    oxc, oxs, oT = oracle.quantize_act(X, inv, L1, r)
    assert np.array_equal(xs.cpu().numpy(), oxs), np.nonzero(xs.cpu().numpy() != oxs)
    assert np.array_equal(xc.cpu().numpy(), oxc), np.nonzero(xc.cpu().numpy() != oxc)
    if r:
        check_T(bf16_to_np_bits(T), oT)
