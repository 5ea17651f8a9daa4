"""The allocation-free activation call (svdq_quantize_act_noalloc).

Some callers of this library cannot allocate device memory or hand it
scratch (a plugin in a host engine that owns every device buffer, serving
code that may not allocate on its request path).  For them the activation
step keeps its scratch in a fixed array inside the library.  These tests call
it through the C ABI, twice in a row, and check that it gives what the
regular call (with a caller workspace) gives: codes and scales byte for
byte, T within the parity tests' tolerance.  The shapes split K over several
CTAs per row tile, so the scratch is really used; a shape whose scratch would
exceed the fixed array is refused before anything runs.

This file is collected last on purpose: it passes alone in a fresh process
and after every other test.
"""

import numpy as np
import pytest

from tests._cases import bf16_to_np_bits, prepare, to_device

pytestmark = pytest.mark.gpu

CASES = [
    ("flux_qkv", 200, 1024, 256, 32),    # 2 row tiles, 16 CTAs per tile
    ("flux_mlp_down", 130, 2048, 128, 64),
    ("sweep_3072", 1, 3072, 128, 16),    # one token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_noalloc_matches_workspace_call_twice(case):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import binding
    from tests.test_gpu_parity import check_T
    p = prepare(*case)
    d = to_device(p)
    assert binding.quantize_act_workspace_bytes(p.M, p.K, p.r) > 0  # the shape uses scratch
    xc, xs, T = svdq.quantize_act(d["X"], d["inv"], d["L1"])
    torch.cuda.synchronize()
    for _ in range(2):
        nc, ns, nT = binding.quantize_act_noalloc(d["X"], d["inv"], d["L1"])
        torch.cuda.synchronize()
        assert svdq.sync_status()[0] == 0
        assert torch.equal(nc, xc)
        assert torch.equal(ns, xs)
        check_T(bf16_to_np_bits(nT), bf16_to_np_bits(T))


def test_noalloc_refuses_shapes_beyond_its_scratch():
    import ctypes
    import torch
    from bit_w4a4_quantized_smooth_b200 import binding
    lib = binding.load()
    M, K, r = 4608, 3072, 128   # needs more scratch than the fixed array holds
    assert binding.quantize_act_workspace_bytes(M, K, r) > (8 << 20)
    P = ctypes.c_void_p
    fake = 0x10000  # never dereferenced: the call refuses on the host first
    rc = lib.svdq_quantize_act_noalloc(P(fake), P(fake), P(fake), M, K, r, P(fake), P(fake), P(fake), None)
    assert rc == 2  # SVDQ_ERR_UNSUPPORTED_SHAPE
    assert torch.cuda.is_available()
