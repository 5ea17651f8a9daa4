"""Smoothing statistics on the device (svdq_channel_absmax) against torch's
own reduction, and the smoothing factors they give against the oracle."""

import numpy as np
import pytest

from tests._cases import bf16_to_np_bits

pytestmark = pytest.mark.gpu


def test_channel_absmax_running_max_over_batches():
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from svdq_inputs import make_layer_inputs
    dev = torch.device("cuda", 0)
    li = make_layer_inputs("flux_qkv", M=777, K=1536, N=256)
    X = torch.from_numpy(li.X.view(np.int16)).view(torch.bfloat16).to(dev)
    # special values in one channel each: -0, +inf, a subnormal, the largest finite
    X[5, 3] = -0.0
    X[700, 9] = float("inf")
    X[1, 17] = 1e-40
    X[2, 18] = -3.3895e38
    amax = torch.zeros(X.shape[1], dtype=torch.float32, device=dev)
    for a, b in ((0, 1), (1, 300), (300, 777)):  # ragged batches, one of a single row
        svdq.channel_absmax(X[a:b], amax)
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    ref = X.abs().amax(dim=0).float()
    assert torch.equal(amax, ref)
    # a second pass over the same rows changes nothing; order does not matter
    amax2 = torch.zeros_like(amax)
    for a, b in ((300, 777), (0, 300)):
        svdq.channel_absmax(X[a:b], amax2)
    assert torch.equal(amax2, amax)


def test_smoothing_from_statistics_matches_oracle(oracle_lib):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import make_layer_inputs
    dev = torch.device("cuda", 0)
    li = make_layer_inputs("flux_qkv", M=640, K=1024, N=512)
    X = torch.from_numpy(li.X.view(np.int16)).view(torch.bfloat16).to(dev)
    W = torch.from_numpy(li.W.view(np.int16)).view(torch.bfloat16).to(dev)
    amax = torch.zeros(li.K, dtype=torch.float32, device=dev)
    for a in range(0, li.M, 128):
        svdq.channel_absmax(X[a:a + 128], amax)
    lam, inv = prep.smoothing_from_stats(amax, W)
    lam_o, inv_o = oracle_lib.smooth(li.X, li.W)
    assert np.array_equal(lam.cpu().numpy(), lam_o)
    assert np.array_equal(inv.cpu().numpy(), inv_o)
