"""Pins of the oracle's GELU (Abramowitz and Stegun 7.1.28 in fp32) and of the
activation step on GELU inputs."""

import math

import numpy as np


def _gelu_exact(x: float) -> float:
    return 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))


def test_within_the_published_bound(oracle_lib):
    # A&S 7.1.28 bounds |erf error| by 3e-7 in exact arithmetic.  In fp32 the
    # 16th power multiplies the rounding error of p (a few 2^-24) by 16, and
    # 1 - 1/p16 turns it into an absolute error of erf: measured below 1.5e-6
    # (near x = -0.06).  Bound: |GELU error| <= 0.5 |x| 2.5e-6, plus ulps of
    # the result; far below bf16's resolution of the activations it feeds.
    xs = np.concatenate([np.linspace(-12, 12, 4801), np.array([1e-6, -1e-6, 0.1, -0.1, 6.5, -6.5])])
    for x in xs.astype(np.float32):
        g = oracle_lib.gelu(float(x))
        ex = _gelu_exact(float(x))
        tol = 0.5 * abs(float(x)) * 2.5e-6 + 4 * np.spacing(np.float32(abs(ex)) + np.float32(1e-38))
        assert abs(g - ex) <= tol, (x, g, ex)


def test_special_values(oracle_lib):
    assert oracle_lib.gelu(0.0) == 0.0
    assert math.copysign(1.0, oracle_lib.gelu(-0.0)) == -1.0
    for x in (8.0, 20.0, 1e6, 3e38):          # erf rounds to 1: GELU(x) = x
        assert oracle_lib.gelu(x) == np.float32(x)
    for x in (-20.0, -1e6, -3e38):            # erf rounds to -1: GELU(x) = -0
        g = oracle_lib.gelu(x)
        assert g == 0.0 and math.copysign(1.0, g) == -1.0
    assert math.isnan(oracle_lib.gelu(float("nan")))
    # the minimum of GELU, near x = -0.7518, value about -0.17
    xs = np.linspace(-1.0, -0.5, 501).astype(np.float32)
    vals = [oracle_lib.gelu(float(x)) for x in xs]
    assert abs(float(xs[int(np.argmin(vals))]) + 0.7518) < 2e-3
    assert abs(min(vals) + 0.16997) < 1e-4


def test_activation_step_on_gelu_inputs(oracle_lib):
    from svdq_inputs import make_layer_inputs
    li = make_layer_inputs("flux_mlp_down", M=5, K=128, N=64, r=16)
    inv = (np.random.default_rng(0).uniform(0.2, 5.0, 128)).astype(np.float32)
    L1 = np.random.default_rng(1).integers(0x3C00, 0x3F80, (128, 16)).astype(np.uint16)
    xc, xs, T = oracle_lib.quantize_act_gelu(li.X, inv, L1, 16)
    # the composition: GELU elementwise in fp32, times inv_lambda (one rounding), then the group quantiser
    x = (li.X.astype(np.uint32) << 16).view(np.float32)
    g = np.array([[oracle_lib.gelu(float(v)) for v in row] for row in x], dtype=np.float32)
    Xh = (g * inv[None, :]).astype(np.float32)
    c2, s2 = oracle_lib.quantize_rows(Xh)
    assert np.array_equal(xc, c2) and np.array_equal(xs, s2)
    # T of the GELU'd, smoothed rows (fp64 sum, one bf16 rounding)
    Xb = (Xh.view(np.uint32) + 0x7FFF + ((Xh.view(np.uint32) >> 16) & 1)) >> 16
    Xbf = (Xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    L1f = (L1.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Tref = np.array([[oracle_lib.bf16_from_f64(v) for v in row] for row in Xbf @ L1f], dtype=np.uint16)
    assert np.array_equal(T, Tref)
    # act = 0 is the plain activation step
    c0, s0, T0 = oracle_lib.quantize_act(li.X, inv, L1, 16)
    assert not np.array_equal(c0, xc)
