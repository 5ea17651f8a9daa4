"""NVFP4 with per-tensor global scales through the C ABI: pre-scaled operands
on the plain calls plus svdq_linear_scaled, against the oracle's two-level
quantiser and linear."""

import numpy as np
import pytest

import oracle
from tests._cases import bf16_bits_to_f64, bf16_to_np_bits

pytestmark = pytest.mark.gpu


def _prepare(M, K, N, r, x_shrink):
    """A layer whose activations are scaled down by `x_shrink` (a power of two):
    without a global scale most activation groups fall below E4M3's range."""
    import torch
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import make_layer_inputs
    li = make_layer_inputs("flux_qkv", M=M, K=K, N=N, r=r)
    X64 = bf16_bits_to_f64(li.X) * x_shrink
    Xb = (X64.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)   # exact: power-of-two shrink
    assert np.array_equal(bf16_bits_to_f64(Xb), X64)
    lam, inv = oracle.smooth(Xb, li.W)
    L1, L2, R, _ = oracle.lowrank(li.W, lam, r)
    dev = torch.device("cuda", 0)
    amax = torch.from_numpy(np.abs(bf16_bits_to_f64(Xb)).max(axis=0).astype(np.float32)).to(dev)
    gx = prep.activation_global_scale(amax, torch.from_numpy(inv).to(dev))
    gw = prep.global_scale(float(np.abs(R).max()))
    return li, Xb, lam, inv, L1, L2, R, gx, gw


@pytest.mark.parametrize("path", ["large", "small"])
@pytest.mark.parametrize("shape", [(200, 512, 272, 32), (64, 1024, 256, 0)], ids=lambda s: "x".join(map(str, s)))
def test_global_scale_layer_matches_oracle(path, shape):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from tests.test_gpu_parity import check_T, rel_fro
    M, K, N, r = shape
    li, Xb, lam, inv, L1, L2, R, gx, gw = _prepare(M, K, N, r, 2.0 ** -14)
    assert gx < 2.0 ** -12  # the activations need the global scale
    dev = torch.device("cuda", 0)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).view(dt).to(dev)
    inv_d = t(inv, torch.float32)
    L1_d = None if r == 0 else t(L1.view(np.int16), torch.bfloat16)
    L2_d = None if r == 0 else t(L2.view(np.int16), torch.bfloat16)
    bias_d = t(li.bias.view(np.int16), torch.bfloat16)
    inv_s, L2_s, R_s, alpha = prep.apply_global_scales(inv_d, L2_d, t(R, torch.float32), gx, gw)
    X_d = t(Xb.view(np.int16), torch.bfloat16)
    rc, rs = svdq.pack_residual(R_s)
    xc, xs, T = svdq.quantize_act(X_d, inv_s, L1_d)
    svdq.set_linear_path(path)
    try:
        Y = svdq.linear(xc, xs, T, rc, rs, L2_s, bias_d, M, K, N, alpha=alpha)
        torch.cuda.synchronize()
    finally:
        svdq.set_linear_path("auto")
    assert svdq.sync_status()[0] == 0
    # the encodings: bit-exact against the oracle's two-level quantiser
    orc, ors = oracle.pack_residual_gs(R, gw)
    oxc, oxs, oT = oracle.quantize_act_gs(Xb, inv, L1, r, gx)
    assert np.array_equal(rc.cpu().numpy(), orc) and np.array_equal(rs.cpu().numpy(), ors)
    assert np.array_equal(xc.cpu().numpy(), oxc) and np.array_equal(xs.cpu().numpy(), oxs)
    if r:
        # the call computed T / g_x (exactly): scaled back it is the oracle's T
        T_back = (T.float() * gx).to(torch.bfloat16)
        assert torch.equal((T_back.float() / gx).to(torch.bfloat16), T)
        check_T(bf16_to_np_bits(T_back), oT)
    Yo = oracle.linear_rows_gs(oxc, oxs, oT, orc, ors, L2, li.bias, M, K, N, r, gx, gw, np.arange(M))
    assert rel_fro(Y.float().cpu().numpy().astype(np.float64), Yo) <= 2e-3


def test_global_scale_keeps_small_activations():
    """The quality statistic: the layer's error against the unquantised
    product, with and without global scales, on tiny activations."""
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    M, K, N, r = 128, 512, 256, 32
    li, Xb, lam, inv, L1, L2, R, gx, gw = _prepare(M, K, N, r, 2.0 ** -16)
    dev = torch.device("cuda", 0)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).view(dt).to(dev)
    X_d = t(Xb.view(np.int16), torch.bfloat16)
    inv_d, L1_d, L2_d = t(inv, torch.float32), t(L1.view(np.int16), torch.bfloat16), t(L2.view(np.int16), torch.bfloat16)
    R_d = t(R, torch.float32)
    ref = (bf16_bits_to_f64(Xb) @ bf16_bits_to_f64(li.W))
    # plain
    rc, rs = svdq.pack_residual(R_d)
    xc, xs, T = svdq.quantize_act(X_d, inv_d, L1_d)
    Y0 = svdq.linear(xc, xs, T, rc, rs, L2_d, None, M, K, N).float().cpu().numpy()
    # global scales
    inv_s, L2_s, R_s, alpha = prep.apply_global_scales(inv_d, L2_d, R_d, gx, gw)
    rc2, rs2 = svdq.pack_residual(R_s)
    xc2, xs2, T2 = svdq.quantize_act(X_d, inv_s, L1_d)
    Y1 = svdq.linear(xc2, xs2, T2, rc2, rs2, L2_s, None, M, K, N, alpha=alpha).float().cpu().numpy()
    torch.cuda.synchronize()
    e0 = np.linalg.norm(Y0 - ref) / np.linalg.norm(ref)
    e1 = np.linalg.norm(Y1 - ref) / np.linalg.norm(ref)
    assert e1 < 0.05, e1        # the usual W4A4 error level
    assert e0 > 4 * e1, (e0, e1)  # without the global scale most groups collapse
