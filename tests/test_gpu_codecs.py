"""The GPU's fp32 -> E2M1 / E4M3 conversions agree with the oracle's codecs.

Runs the real residual packer on crafted inputs: every group holds one
element equal to 6 * t, which makes the scale E4M3(RN(t)) and, for t = 1,
rcp = 1, so the other 15 elements are converted to E2M1 as they are.  The
sweep covers every fp32 value with at most 10 mantissa bits in [-6, 6], the
neighbours of every rounding tie, signed zeros and random values; the scale
sweep covers [2^-12, 600].  Any disagreement in rounding, tie breaking,
saturation or the sign of zero fails the byte comparison.
"""

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def _pack_both(groups: np.ndarray):
    """groups [G][16] fp32 -> compare GPU and oracle packing of R = groups^T."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    G = groups.shape[0]
    n_cols = -(-G // 4)
    n_cols = -(-n_cols // 16) * 16
    flat = np.zeros((n_cols * 4, 16), dtype=np.float32)
    flat[:G] = groups
    # group i = 4 n + g sits in rows [16 g, 16 g + 16) of column n
    R = np.ascontiguousarray(flat.reshape(n_cols, 4, 16).transpose(1, 2, 0).reshape(64, n_cols))
    rc, rs = svdq.pack_residual(torch.from_numpy(R).cuda())
    torch.cuda.synchronize()
    orc, ors = oracle.pack_residual(R)
    return rc.cpu().numpy(), rs.cpu().numpy(), orc, ors


def _grid_values():
    vals = set()
    for e in range(-10, 3):            # magnitudes 2^-10 .. 7.99
        for m in range(1024):
            v = (1.0 + m / 1024.0) * 2.0 ** e
            if v <= 6.0:
                vals.add(v)
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for t in ties:
        f = np.float32(t)
        vals.update([float(np.nextafter(f, np.float32(0))), float(f), float(np.nextafter(f, np.float32(9)))])
    vals = sorted(vals)
    out = np.array(vals + [-v for v in vals] + [0.0, -0.0, 1e-30, -1e-30, -1e-9], dtype=np.float32)
    rng = np.random.default_rng(0)
    return np.concatenate([out, rng.uniform(-6, 6, 200000).astype(np.float32)])


def test_e2m1_conversion_matches_oracle():
    v = _grid_values()
    per = 15
    G = -(-len(v) // per)
    body = np.zeros(G * per, dtype=np.float32)
    body[: len(v)] = v
    groups = np.concatenate([np.full((G, 1), 6.0, np.float32), body.reshape(G, per)], axis=1)
    rc, rs, orc, ors = _pack_both(groups)
    assert np.array_equal(rs, ors)
    mism = np.nonzero(rc != orc)
    assert mism[0].size == 0, f"{mism[0].size} code bytes differ"


def test_e4m3_scale_conversion_matches_oracle():
    ts = set()
    for e in range(-12, 10):
        for m in range(0, 1024, 3):
            t = (1.0 + m / 1024.0) * 2.0 ** e
            if t <= 600:
                ts.add(t)
    ts = np.array(sorted(ts), dtype=np.float32)
    rng = np.random.default_rng(1)
    ts = np.concatenate([ts, (10.0 ** rng.uniform(-4, 2.8, 20000)).astype(np.float32)])
    groups = np.zeros((len(ts), 16), dtype=np.float32)
    groups[:, 0] = 6.0 * ts
    groups[:, 1] = -3.0 * ts
    groups[:, 2] = 0.7 * ts
    groups[:, 3] = -0.01 * ts
    rc, rs, orc, ors = _pack_both(groups)
    assert np.array_equal(rs, ors)
    assert np.array_equal(rc, orc)
