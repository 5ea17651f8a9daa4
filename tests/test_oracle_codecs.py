"""Pins for the oracle's scalar codecs (bf16, E4M3, E2M1) and group quantiser.

Each check compares the oracle with something other than itself: the
published format tables (golden files), torch's own float8/bfloat16 casts,
brute-force nearest-value search over the whole grid, and hand-worked groups.
"""

import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ E4M3 ----

def test_e4m3_decode_all_codes_match_torch(oracle_lib):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle_lib.e4m3_decode(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v) and math.isnan(ref[c])
        else:
            assert v == ref[c], (hex(c), v, ref[c])
            assert math.copysign(1.0, v) == math.copysign(1.0, ref[c])


def test_e4m3_special_values(oracle_lib):
    for code, val in _read_table("e4m3_special.txt"):
        c, v = int(code, 16), float(val)
        assert oracle_lib.e4m3_decode(c) == v
        assert oracle_lib.e4m3_encode(v) == c


def _e4m3_grid():
    vals = [(c, torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).item()) for c in range(0x7F)]
    return vals  # non-negative finite codes 0x00..0x7E, ascending


def _e4m3_brute(x):
    """Nearest non-negative E4M3 value by exhaustive search, ties to even code."""
    a = abs(x)
    if a >= 448.0:
        return 0x7E
    best = None
    for c, v in _e4m3_grid():
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return best[1]


def test_e4m3_encode_matches_brute_force_and_torch(oracle_lib):
    rng = np.random.default_rng(1)
    xs = list(np.float32(10.0) ** rng.uniform(-4, 2.7, 3000).astype(np.float32))
    grid = [v for _, v in _e4m3_grid()]
    xs += [np.float32((a + b) / 2) for a, b in zip(grid[:-1], grid[1:])]  # every midpoint
    xs += [np.float32(v) for v in grid]
    for x in xs:
        x = float(np.float32(x))
        got = oracle_lib.e4m3_encode(x)
        assert got == _e4m3_brute(x), x
        if x < 464.0:  # torch rounds without saturation; compare inside the range
            t = torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item()
            assert got == t, (x, got, t)


def test_e4m3_saturates(oracle_lib):
    for x in [448.0, 449.0, 464.0, 465.0, 1e6, 3.0e38]:
        assert oracle_lib.e4m3_encode(x) == 0x7E
    assert oracle_lib.e4m3_encode(-1e6) == 0xFE


def test_e4m3_round_trip_every_finite_value(oracle_lib):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = oracle_lib.e4m3_decode(c)
        assert oracle_lib.e4m3_encode(v) == c


# ------------------------------------------------------------------ E2M1 ----

def test_e2m1_table(oracle_lib):
    for row in _read_table("e2m1_table.txt"):
        if row[0] in ("tie", "sat"):
            x, code = float(row[1]), int(row[2], 16)
            assert oracle_lib.e2m1_encode(x) == code, row
        else:
            code, v = int(row[0], 16), float(row[1])
            got = oracle_lib.e2m1_decode(code)
            assert got == v and math.copysign(1, got) == math.copysign(1, v)
            assert oracle_lib.e2m1_encode(v) == code


def _e2m1_brute(x):
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    a = abs(x)
    best = None
    for c, v in enumerate(grid):
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    c = best[1]
    return c | (8 if math.copysign(1.0, x) < 0 else 0)


def test_e2m1_encode_matches_brute_force(oracle_lib):
    rng = np.random.default_rng(2)
    xs = list(rng.uniform(-8, 8, 20000).astype(np.float32))
    # every float with <= 10 mantissa bits in [-8, 8] on a coarse lattice
    xs += list(np.arange(-8.0, 8.0, 1.0 / 64, dtype=np.float32))
    xs += [np.float32(-0.0), np.float32(0.0), np.float32(-1e-30), np.float32(1e-30)]
    for x in xs:
        x = float(x)
        assert oracle_lib.e2m1_encode(x) == _e2m1_brute(x), x


# ------------------------------------------------------------------ bf16 ----

def test_bf16_from_fp32_matches_torch(oracle_lib):
    rng = np.random.default_rng(3)
    xs = (rng.standard_normal(5000) * 10.0 ** rng.uniform(-20, 20, 5000)).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    for x, r in zip(xs, ref):
        assert oracle_lib.bf16_from_f64(float(x)) == r, x


def test_bf16_from_f64_is_nearest_even(oracle_lib):
    rng = np.random.default_rng(4)
    xs = rng.standard_normal(3000) * 10.0 ** rng.uniform(-5, 5, 3000)
    for x in xs:
        b = oracle_lib.bf16_from_f64(float(x))
        v = oracle_lib.bf16_to_f32(b)
        # neighbours on the bf16 grid (same sign, adjacent bit patterns)
        lo = oracle_lib.bf16_to_f32((b - 1) & 0xFFFF)
        hi = oracle_lib.bf16_to_f32((b + 1) & 0xFFFF)
        d = abs(x - v)
        assert d <= abs(x - lo) and d <= abs(x - hi)
        if d == abs(x - lo) or d == abs(x - hi):
            assert b % 2 == 0


# -------------------------------------------------------- group quantiser ----

def test_worked_groups(oracle_lib):
    for row in _read_table("nvfp4_groups.txt"):
        line = " ".join(row)
        vals, sc, codes = [p.split() for p in line.split("|")]
        v = np.array([float(t) for t in vals], dtype=np.float32)
        got_codes, got_s = oracle_lib.quantize_group(v)
        assert got_s == int(sc[0], 16), line
        assert [int(c) for c in got_codes] == [int(c, 16) for c in codes], line


def test_group_error_bound(oracle_lib):
    """|v - deq(q)| <= s_d for every element; s_d within 2^-4 of amax/6
    when amax/6 is in E4M3's normal range and below the saturation point."""
    rng = np.random.default_rng(5)
    for _ in range(400):
        scale = 10.0 ** rng.uniform(-1.5, 2.0)
        v = (rng.standard_normal(16) * scale).astype(np.float32)
        codes, s = oracle_lib.quantize_group(v)
        sd = oracle_lib.e4m3_decode(s)
        amax = float(np.max(np.abs(v)))
        target = amax / 6.0
        if 2.0 ** -6 <= target <= 448.0:
            assert abs(sd - target) <= target * 2.0 ** -4 * 1.0000001
        for x, c in zip(v, codes):
            d = oracle_lib.e2m1_decode(int(c)) * sd
            assert abs(float(x) - d) <= sd * 1.0000001, (x, d, sd)


def test_zero_group(oracle_lib):
    v = np.zeros(16, dtype=np.float32)
    v[3] = -0.0
    codes, s = oracle_lib.quantize_group(v)
    assert s == 0
    assert list(codes) == [0, 0, 0, 8] + [0] * 12
