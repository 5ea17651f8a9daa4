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
    # widest K first, then narrower (stale tails must not leak), and an MLP
    # pair (2 -> 3): layer 3 reads GELU of layer 2's output
    ids = [77, 0, 76, 1, 2, 3, 4]
    layers = bench.prepare_stack(device, M=M, layer_ids=ids)
    assert [L["gelu"] for L in layers] == [False, False, False, False, False, True, False]
    ref = []
    for L in layers:
        X = ref[-1] if L["gelu"] else L["X"]
        xc, xs, T = svdq.quantize_act(X, L["inv"], L["L1"], gelu=L["gelu"])
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
