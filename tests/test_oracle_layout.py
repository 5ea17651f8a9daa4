"""Pins for the oracle's packed layouts (code nibbles and 128x4 scale tiles)."""

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_scale_offsets_hand_computed(oracle_lib):
    with open(os.path.join(GOLDEN, "scale_layout.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            K, row, g, off = (int(t) for t in line.split())
            assert oracle_lib.scale_offset(row, g, K) == off, line


def test_scale_layout_is_a_bijection(oracle_lib):
    for rows, K in [(1, 64), (128, 64), (200, 192), (256, 1024)]:
        padded = ((rows + 127) // 128) * 128
        total = oracle_lib.scale_bytes(rows, K)
        assert total == padded * K // 16
        seen = np.zeros(total, dtype=np.int32)
        for r in range(padded):
            for g in range(K // 16):
                seen[oracle_lib.scale_offset(r, g, K)] += 1
        assert np.all(seen == 1)


def test_code_nibble_order(oracle_lib):
    """Element k of a row lands in byte k/2, low nibble for even k."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    # magnitude grid[k % 8], negative on odd octets (so -0.0 appears too);
    # every group of 16 holds a +-6, so each scale is exactly 1.0 (0x38)
    v = np.array([[grid[k % 8] * (-1.0 if (k // 8) % 2 else 1.0) for k in range(64)]],
                 dtype=np.float32)
    codes, scales = oracle_lib.quantize_rows(v)
    for k in range(64):
        expect = (k % 8) | (8 if (k // 8) % 2 else 0)
        byte = int(codes[0, k // 2])
        got = (byte >> 4) if (k & 1) else (byte & 15)
        assert got == expect, (k, got, expect)
    for g in range(4):
        assert scales[oracle_lib.scale_offset(0, g, 64)] == 0x38


def test_quantize_rows_equals_groupwise(oracle_lib):
    rng = np.random.default_rng(7)
    V = (rng.standard_normal((37, 192)) * 3).astype(np.float32)
    codes, scales = oracle_lib.quantize_rows(V)
    deq = oracle_lib.dequant(codes, scales, 37, 192)
    for i in range(37):
        for g in range(12):
            c, s = oracle_lib.quantize_group(V[i, g * 16:(g + 1) * 16])
            sd = oracle_lib.e4m3_decode(s)
            ref = np.array([oracle_lib.e2m1_decode(int(x)) * sd for x in c])
            assert np.array_equal(deq[i, g * 16:(g + 1) * 16].astype(np.float64), ref)
            assert scales[oracle_lib.scale_offset(i, g, 192)] == s
    # padding rows of the last 128-row band hold zero scales
    for i in range(37, 128):
        for g in range(12):
            assert scales[oracle_lib.scale_offset(i, g, 192)] == 0


def test_pack_residual_is_column_quantisation(oracle_lib):
    rng = np.random.default_rng(8)
    R = (rng.standard_normal((128, 24)) * 0.02).astype(np.float32)
    rc, rs = oracle_lib.pack_residual(R)
    c2, s2 = oracle_lib.quantize_rows(np.ascontiguousarray(R.T))
    assert np.array_equal(rc, c2) and np.array_equal(rs, s2)
