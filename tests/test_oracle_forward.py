"""Pins for the oracle's quantised forward (activation step + linear).

Brute force on tiny inputs rebuilds every output element with plain Python
loops from the separately pinned scalar codecs (group quantiser, E2M1/E4M3
decode, bf16 rounding), so a dropped term, a wrong index or a transposed
operand anywhere in the packed path fails here.
"""

import numpy as np
import pytest
import torch

from svdq_inputs import bf16_bits_to_f32, make_layer_inputs


def _prep(oracle_lib, li, r, smooth=True):
    if smooth:
        lam, inv = oracle_lib.smooth(li.Xcal, li.W)
    else:
        lam = np.ones(li.K, dtype=np.float32)
        inv = np.ones(li.K, dtype=np.float32)
    L1, L2, R, _ = oracle_lib.lowrank(li.W, lam, r)
    return lam, inv, L1, L2, R


def _group_deq(oracle_lib, v):
    codes, s = oracle_lib.quantize_group(v)
    sd = oracle_lib.e4m3_decode(s)
    return [oracle_lib.e2m1_decode(int(c)) * sd for c in codes]


@pytest.mark.parametrize("M,K,N,r,bias", [(5, 64, 7, 16, True), (3, 128, 4, 0, False),
                                          (2, 64, 3, 32, True)])
def test_forward_brute_force(oracle_lib, M, K, N, r, bias):
    li = make_layer_inputs("flux_qkv" if bias else "tiny", M=M, K=K, N=N, r=r)
    lam, inv, L1, L2, R = _prep(oracle_lib, li, r)
    xc, xs, T = oracle_lib.quantize_act(li.X, inv, L1, r)
    rc, rs = oracle_lib.pack_residual(R)
    Y = oracle_lib.linear_rows(xc, xs, T, rc, rs, L2 if r else None, li.bias, M, K, N, r,
                               np.arange(M))
    # --- brute force ---
    Xh = bf16_bits_to_f32(li.X) * inv[None, :]          # numpy fp32 products
    xdeq = [sum((_group_deq(oracle_lib, Xh[m, g * 16:(g + 1) * 16]) for g in range(K // 16)), [])
            for m in range(M)]
    rdeq = [sum((_group_deq(oracle_lib, np.ascontiguousarray(R[g * 16:(g + 1) * 16, n]))
                 for g in range(K // 16)), []) for n in range(N)]
    Xb = torch.from_numpy(Xh).to(torch.bfloat16).double().numpy()   # bf16(Xh)
    L1d = bf16_bits_to_f32(L1).astype(np.float64) if r else None
    L2d = bf16_bits_to_f32(L2).astype(np.float64) if r else None
    bd = bf16_bits_to_f32(li.bias).astype(np.float64) if bias else np.zeros(N)
    for m in range(M):
        Tm = []
        for j in range(r):
            acc = 0.0
            for k in range(K):
                acc += float(Xb[m, k]) * float(L1d[k, j])
            Tm.append(oracle_lib.bf16_to_f32(oracle_lib.bf16_from_f64(acc)))
        if r:
            assert np.array_equal(bf16_bits_to_f32(T[m]).astype(np.float64), np.array(Tm))
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += xdeq[m][k] * rdeq[n][k]
            for j in range(r):
                acc += Tm[j] * float(L2d[j, n])
            acc += bd[n]
            assert Y[m, n] == pytest.approx(acc, rel=1e-13, abs=1e-13)


def test_dequant_matches_groups(oracle_lib):
    li = make_layer_inputs("tiny", M=4, K=128, N=32, r=0)
    lam, inv, L1, L2, R = _prep(oracle_lib, li, 0)
    rc, rs = oracle_lib.pack_residual(R)
    Rd = oracle_lib.dequant(rc, rs, 32, 128)
    for n in range(0, 32, 7):
        for g in range(8):
            ref = _group_deq(oracle_lib, np.ascontiguousarray(R[g * 16:(g + 1) * 16, n]))
            assert np.array_equal(Rd[n, g * 16:(g + 1) * 16].astype(np.float64), np.array(ref))


def _rel_err(Y, ref):
    return float(np.linalg.norm(Y - ref) / np.linalg.norm(ref))


def test_quality_ordering(oracle_lib):
    """Quantisation error of the four variants on the tiny workload's shape.

    The pages claim smoothing alone is not enough at 4 bits and that the
    low-rank branch absorbs the outliers (ai-digest.ru SVDQuant abstract), so
    SVDQuant must beat smoothing-only and naive W4A4, and the low-rank branch
    alone must beat naive W4A4.  These are reported statistics, not parity.
    """
    li = make_layer_inputs("tiny", M=128, K=512, N=256, r=16)
    X = bf16_bits_to_f32(li.X).astype(np.float64)
    W = bf16_bits_to_f32(li.W).astype(np.float64)
    ref = X @ W
    errs = {}
    for name, smooth, r in [("svdquant", True, 16), ("smooth_only", True, 0),
                            ("lowrank_only", False, 16), ("naive", False, 0)]:
        lam, inv, L1, L2, R = _prep(oracle_lib, li, r, smooth)
        xc, xs, T = oracle_lib.quantize_act(li.X, inv, L1, r)
        rc, rs = oracle_lib.pack_residual(R)
        Y = oracle_lib.linear_rows(xc, xs, T, rc, rs, L2 if r else None, None, li.M, li.K, li.N, r,
                                   np.arange(li.M))
        errs[name] = _rel_err(Y, ref)
    print("relative Frobenius error vs X W:", errs)
    assert errs["svdquant"] < errs["smooth_only"]
    assert errs["svdquant"] < errs["naive"]
    assert errs["lowrank_only"] < errs["naive"]
    assert errs["svdquant"] < 0.2
