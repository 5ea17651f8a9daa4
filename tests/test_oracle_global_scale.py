"""Pins of the oracle's NVFP4 quantiser with a per-tensor global scale
(two-level scaling: q * decode(s) * g)."""

import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_global_scale.txt")


def _rows():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        vals, g, s, codes = [p.strip() for p in line.split("|")]
        yield (np.array([float(x) for x in vals.split()], dtype=np.float32), float(g), int(s, 16),
               np.array([int(c, 16) for c in codes.split()], dtype=np.uint8))


def test_hand_worked_groups(oracle_lib):
    rows = list(_rows())
    assert len(rows) == 4
    for v, g, s, codes in rows:
        c, sc = oracle_lib.quantize_group_gs(v, g)
        assert sc == s, (v, g)
        assert np.array_equal(c, codes), (v, g, c)


def _groups(n, seed):
    rng = np.random.default_rng(seed)
    mags = 10.0 ** rng.uniform(-5, 3, size=(n, 1))
    return (rng.standard_normal((n, 16)) * mags).astype(np.float32)


def test_unit_global_scale_is_the_plain_quantiser(oracle_lib):
    for v in _groups(400, 1):
        assert oracle_lib.quantize_group_gs(v, 1.0)[1] == oracle_lib.quantize_group(v)[1]
        assert np.array_equal(oracle_lib.quantize_group_gs(v, 1.0)[0], oracle_lib.quantize_group(v)[0])


def test_power_of_two_scaling_invariance(oracle_lib):
    # scaling the values and g by the same power of two changes nothing
    rng = np.random.default_rng(2)
    for v in _groups(200, 3):
        g = float(2.0 ** rng.integers(-14, 6)) * float(rng.uniform(0.5, 1.0))
        j = int(rng.integers(-8, 9))
        a = oracle_lib.quantize_group_gs(v, g)
        b = oracle_lib.quantize_group_gs((v * np.float32(2.0 ** j)).astype(np.float32), g * 2.0 ** j)
        assert a[1] == b[1] and np.array_equal(a[0], b[0])


def test_power_of_two_global_scale_equals_plain_on_the_scaled_group(oracle_lib):
    # for g = 2^e the two-level encoding of v is the plain encoding of v / g
    # (every step is an exact scaling by a power of two): the identity that
    # lets the plain kernels serve the variant on pre-scaled operands
    rng = np.random.default_rng(4)
    for v in _groups(400, 5):
        e = int(rng.integers(-16, 8))
        a = oracle_lib.quantize_group_gs(v, 2.0 ** e)
        b = oracle_lib.quantize_group((v * np.float32(2.0 ** -e)).astype(np.float32))
        assert a[1] == b[1] and np.array_equal(a[0], b[0])


def test_error_bound_inside_the_range(oracle_lib):
    # with the group's scale in E4M3's normal range, |v - q d| <= d
    rng = np.random.default_rng(6)
    checked = 0
    for v in _groups(600, 7):
        amax = float(np.abs(v).max())
        g = amax / (6.0 * float(rng.uniform(1.0, 400.0)))   # scale lands in [1, 400]
        codes, s = oracle_lib.quantize_group_gs(v, g)
        d = float(np.float32(oracle_lib.e4m3_decode(s) * np.float32(g)))
        q = np.array([oracle_lib.e2m1_decode(int(c)) for c in codes])
        assert np.all(np.abs(v.astype(np.float64) - q * d) <= d * (1 + 1e-6) + 1e-30)
        checked += 1
    assert checked == 600


def test_rows_pack_and_activation_match_the_group_quantiser(oracle_lib):
    rng = np.random.default_rng(8)
    K, N, g = 128, 32, 2.0 ** -7
    R = (rng.standard_normal((K, N)) * 1e-3).astype(np.float32)
    rc, rs = oracle_lib.pack_residual_gs(R, g)
    for n in (0, 7, 31):
        for grp in (0, 5):
            codes, s = oracle_lib.quantize_group_gs(R[16 * grp:16 * grp + 16, n], g)
            assert rs[oracle_lib.scale_offset(n, grp, K)] == s
            packed = rc[n, 8 * grp:8 * grp + 8]
            assert np.array_equal(packed & 15, codes[0::2]) and np.array_equal(packed >> 4, codes[1::2])
    V = R.T.copy()
    c2, s2 = oracle_lib.quantize_rows_gs(V, g)
    assert np.array_equal(c2, rc) and np.array_equal(s2, rs)


def test_linear_with_global_scales(oracle_lib):
    from svdq_inputs import make_layer_inputs
    li = make_layer_inputs("flux_qkv", M=6, K=128, N=48, r=16)
    lam, inv = oracle_lib.smooth(li.X, li.W)
    L1, L2, R, _ = oracle_lib.lowrank(li.W, lam, 16)
    gx, gw = 2.0 ** -3, 2.0 ** -9
    xc, xs, T = oracle_lib.quantize_act_gs(li.X, inv, L1, 16, gx)
    xc1, xs1, T1 = oracle_lib.quantize_act(li.X, inv, L1, 16)
    assert np.array_equal(T, T1)  # T is of Xh itself
    rc, rs = oracle_lib.pack_residual_gs(R, gw)
    rows = np.arange(6)
    Y = oracle_lib.linear_rows_gs(xc, xs, T, rc, rs, L2, li.bias, 6, 128, 48, 16, gx, gw, rows)
    Ylr = oracle_lib.linear_rows_gs(xc, xs, T, rc, rs, L2, li.bias, 6, 128, 48, 16, 1.0, 1.0, rows)
    Y0 = oracle_lib.linear_rows(xc, xs, T, rc, rs, L2, li.bias, 6, 128, 48, 16, rows)
    assert np.array_equal(Ylr, Y0)
    # only the 4-bit product carries the global scales
    Ylow = oracle_lib.linear_rows(xc, xs, T, np.zeros_like(rc), np.zeros_like(rs), L2, li.bias, 6, 128, 48,
                                  16, rows)
    assert np.allclose(Y - Ylow, gx * gw * (Y0 - Ylow), rtol=1e-12, atol=0)
