"""LoRA adapters joined to the low-rank branch without re-quantising R.

With Xh = X diag(lambda)^-1, an adapter (A [K][ra], B [ra][N]) joins as
L1' = [L1 | bf16(RN_f32(lambda A))], L2' = [L2 ; B]: Xh L1' L2' = Xh L1 L2 +
X A B, and the 4-bit residual stays as packed (chattools.cn
"SVDQuant的主要功能", item LoRA集成).
"""

import numpy as np
import pytest

import oracle
from svdq_inputs import make_layer_inputs
from svdq_inputs.workloads import make_lora  # noqa: E402
from tests._cases import bf16_bits_to_f64, prepare

CASE = ("flux_qkv", 200, 320, 272, 32)
RA = 32


def _lora(p):
    return make_lora(0x5EED7000, p.K, p.N, RA)


def test_attach_layout_is_concatenation():
    p = prepare(*CASE)
    A, B = _lora(p)
    L1n, L2n = oracle.attach_lora(p.L1, p.L2, p.lam, A, B)
    assert L1n.shape == (p.K, p.r + RA) and L2n.shape == (p.r + RA, p.N)
    assert np.array_equal(L1n[:, :p.r], p.L1)
    assert np.array_equal(L2n[:p.r], p.L2)
    assert np.array_equal(L2n[p.r:], B)


def test_smoothing_cancels_on_the_adapter_columns():
    """Xh (lambda A) = X A up to the rounding of lambda A to bf16 (2^-9
    relative per entry) and of Xh to fp32: a missing or inverted lambda
    fails by orders of magnitude."""
    p = prepare(*CASE)
    A, B = _lora(p)
    L1n, _ = oracle.attach_lora(p.L1, p.L2, p.lam, A, B)
    X = bf16_bits_to_f64(p.X)
    Xh = (X.astype(np.float32) * p.inv).astype(np.float64)
    got = Xh @ bf16_bits_to_f64(L1n[:, p.r:])
    want = X @ bf16_bits_to_f64(A)
    err = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err < 2.0 ** -8, err
    # the same check with lambda left out is far off
    bad = Xh @ bf16_bits_to_f64(A)
    assert np.linalg.norm(bad - want) / np.linalg.norm(want) > 0.1


def test_product_prep_matches_oracle_bit_exact():
    torch = pytest.importorskip("torch")
    from bit_w4a4_quantized_smooth_b200 import prep
    p = prepare(*CASE)
    A, B = _lora(p)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    L1t, L2t = prep.attach_lora(t(p.L1), t(p.L2), torch.from_numpy(p.lam), t(A), t(B))
    L1n, L2n = oracle.attach_lora(p.L1, p.L2, p.lam, A, B)
    assert np.array_equal(L1t.view(torch.int16).numpy().view(np.uint16), L1n)
    assert np.array_equal(L2t.view(torch.int16).numpy().view(np.uint16), L2n)


def test_layer_adds_x_a_b():
    """The oracle's layer with the joined factors minus the layer without
    them is X A B, up to T's bf16 rounding."""
    p = prepare(*CASE)
    A, B = _lora(p)
    L1n, L2n = oracle.attach_lora(p.L1, p.L2, p.lam, A, B)
    rc, rs = oracle.pack_residual(p.R)
    rows = np.arange(p.M)
    xc, xs, T0 = oracle.quantize_act(p.X, p.inv, p.L1, p.r)
    Y0 = oracle.linear_rows(xc, xs, T0, rc, rs, p.L2, p.bias, p.M, p.K, p.N, p.r, rows)
    xc1, xs1, T1 = oracle.quantize_act(p.X, p.inv, L1n, p.r + RA)
    assert np.array_equal(xc1, xc) and np.array_equal(xs1, xs)   # the 4-bit path is untouched
    Y1 = oracle.linear_rows(xc, xs, T1, rc, rs, L2n, p.bias, p.M, p.K, p.N, p.r + RA, rows)
    delta = Y1 - Y0
    want = bf16_bits_to_f64(p.X) @ bf16_bits_to_f64(A) @ bf16_bits_to_f64(B)
    err = np.linalg.norm(delta - want) / np.linalg.norm(want)
    assert err < 1e-2, err


@pytest.mark.gpu
def test_gpu_layer_with_lora_matches_oracle():
    """The joined factors through the C ABI (rank 32 + 32 = 64)."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from tests._cases import to_device, bf16_to_np_bits
    from tests.test_gpu_parity import check_T, rel_fro, Y_TOL
    svdq.load()
    p = prepare(*CASE)
    A, B = _lora(p)
    L1n, L2n = oracle.attach_lora(p.L1, p.L2, p.lam, A, B)
    d = to_device(p)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    rc, rs = svdq.pack_residual(d["R"])
    xc, xs, T = svdq.quantize_act(d["X"], d["inv"], bf(L1n))
    Y = svdq.linear(xc, xs, T, rc, rs, bf(L2n), d["bias"], p.M, p.K, p.N)
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    r2 = p.r + RA
    oxc, oxs, oT = oracle.quantize_act(p.X, p.inv, L1n, r2)
    orc, ors = oracle.pack_residual(p.R)
    assert np.array_equal(xc.cpu().numpy(), oxc) and np.array_equal(xs.cpu().numpy(), oxs)
    check_T(bf16_to_np_bits(T), oT)
    ref = oracle.linear_rows(oxc, oxs, oT, orc, ors, L2n, p.bias, p.M, p.K, p.N, r2, np.arange(p.M))
    err = rel_fro(bf16_bits_to_f64(bf16_to_np_bits(Y)), ref)
    assert err <= Y_TOL, err


@pytest.mark.gpu
@pytest.mark.parametrize("r", [0, 32])
def test_gpu_attach_lora_matches_oracle_bit_exact(r):
    """svdq_attach_lora (device-side join) equals the oracle's join bit for
    bit, also with no SVD branch (r = 0) and with a second adapter chained
    onto the first."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    p = prepare(*CASE)
    L1 = p.L1 if r else None
    L2 = p.L2 if r else None
    A, B = _lora(p)
    A2, B2 = make_lora(0x5EED7001, p.K, p.N, 16)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    bits = lambda x: x.cpu().view(torch.int16).numpy().view(np.uint16)
    lam = torch.from_numpy(p.lam).cuda()
    L1g, L2g = svdq.attach_lora(t(L1), t(L2), lam, t(A), t(B))
    L1h, L2h = svdq.attach_lora(L1g, L2g, lam, t(A2), t(B2))
    torch.cuda.synchronize()
    L1n, L2n = oracle.attach_lora(L1, L2, p.lam, A, B)
    L1m, L2m = oracle.attach_lora(L1n, L2n, p.lam, A2, B2)
    assert np.array_equal(bits(L1g), L1n) and np.array_equal(bits(L2g), L2n)
    assert np.array_equal(bits(L1h), L1m) and np.array_equal(bits(L2h), L2m)
