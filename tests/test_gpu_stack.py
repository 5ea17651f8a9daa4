"""The DiT-stack pass of bench.py: layers sharing activation buffers in one
stream (and replayed from a CUDA graph) give what each layer gives alone."""

import pytest

pytestmark = pytest.mark.gpu


def test_stack_pass_matches_layers_alone():
    import torch
    import bench
    import bit_w4a4_quantized_smooth_b200 as svdq
    device = torch.device("cuda", 0)
    M = 200  # two activation row tiles, ragged
    ids = [3, 0, 77, 1, 76, 2]  # widest K first, then narrower: stale tails must not leak
    layers = bench.prepare_stack(device, M=M, layer_ids=ids)
    ref = []
    for L in layers:
        xc, xs, T = svdq.quantize_act(L["X"], L["inv"], L["L1"])
        ref.append(svdq.linear(xc, xs, T, L["rc"], L["rs"], L["L2"], None, M, L["K"], L["N"]))
    Y = [torch.full((M, L["N"]), float("nan"), dtype=torch.bfloat16, device=device) for L in layers]
    run = bench.stack_pass_fn(layers, device, M=M, Y_out=Y)
    run()
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    for i, (a, b) in enumerate(zip(Y, ref)):
        assert torch.equal(a, b), ids[i]
    # the same pass replayed from a CUDA graph
    for y in Y:
        y.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g):
        run()
    for y in Y:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert svdq.sync_status()[0] == 0
    for i, (a, b) in enumerate(zip(Y, ref)):
        assert torch.equal(a, b), ids[i]
    del g
