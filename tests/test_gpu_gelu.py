"""The activation step on GELU inputs (svdq_quantize_act_gelu) against the
oracle: codes and scales bit-exact, T within the parity tolerance, and the
layer's output through the linear call."""

import numpy as np
import pytest

import oracle
from tests._cases import bf16_to_np_bits

pytestmark = pytest.mark.gpu

CASES = [
    ("flux_qkv", 200, 512, 256, 32),      # outlier channels (large |x|), ragged M
    ("flux_mlp_up", 130, 2048, 128, 64),  # K split over CTAs, two rank atoms
    ("flux_mlp_up", 1, 1024, 256, 16),    # one token
    ("flux_mlp_up", 512, 12288, 256, 32), # the MLP down-projection's K
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_gelu_activation_step_matches_oracle(case):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from svdq_inputs import make_layer_inputs
    from tests.test_gpu_parity import check_T, rel_fro
    name, M, K, N, r = case
    li = make_layer_inputs(name, M=M, K=K, N=N, r=r)
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(7)
    inv = rng.uniform(0.1, 4.0, K).astype(np.float32)
    L1 = (0.05 * rng.standard_normal((K, r))).astype(np.float32)
    L1b = ((L1.view(np.uint32) + 0x7FFF + ((L1.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16)
    X = torch.from_numpy(li.X.view(np.int16)).view(torch.bfloat16).to(dev)
    xc, xs, T = svdq.quantize_act(X, torch.from_numpy(inv).to(dev),
                                  torch.from_numpy(L1b.view(np.int16)).view(torch.bfloat16).to(dev), gelu=True)
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    oxc, oxs, oT = oracle.quantize_act_gelu(li.X, inv, L1b, r)
    assert np.array_equal(xc.cpu().numpy(), oxc)
    assert np.array_equal(xs.cpu().numpy(), oxs)
    check_T(bf16_to_np_bits(T), oT)
    # through the linear call: the layer on GELU inputs
    W = li.W
    R = (0.02 * rng.standard_normal((K, N))).astype(np.float32)
    rc, rs = svdq.pack_residual(torch.from_numpy(R).to(dev))
    L2 = (0.05 * rng.standard_normal((r, N))).astype(np.float32)
    L2b = ((L2.view(np.uint32) + 0x7FFF + ((L2.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16)
    Y = svdq.linear(xc, xs, T, rc, rs, torch.from_numpy(L2b.view(np.int16)).view(torch.bfloat16).to(dev), None,
                    M, K, N)
    orc, ors = oracle.pack_residual(R)
    rows = np.arange(min(M, 64))
    Yo = oracle.linear_rows(oxc, oxs, oT, orc, ors, L2b, None, M, K, N, r, rows)
    assert rel_fro(Y.float().cpu().numpy()[rows].astype(np.float64), Yo) <= 2e-3
