"""Launch overlap (programmatic dependent launch) keeps stream order for every
buffer the layer calls share with the kernels around them.

One stream, no host synchronisation: a torch kernel rewrites X right before
the activation call, the residual packer rewrites R right before the linear
call (whose kernels prefetch R into L2 before they wait), a torch kernel reads
Y right after it, and a second layer reads the first layer's Y as its X.  The
outputs are bit-identical to the same sequence launched plainly with a device
synchronisation after every call, and to a CUDA graph of it; the first
output matches the oracle."""

import numpy as np
import pytest

import oracle
from tests._cases import bf16_to_np_bits, prepare, to_device

pytestmark = pytest.mark.gpu

# (workload, M, K, N, N2, r): the small-M split-K kernel, then the large-M pair kernel
CASES = [
    ("flux_qkv", 64, 1024, 512, 256, 32),
    ("flux_qkv", 520, 1024, 768, 512, 32),
]


def _sequence(svdq, torch, bufs, A, B, steps, sync):
    """The calls of `steps` iterations on the current stream -> the Y copies."""
    outs = []
    for i in range(steps):
        bufs["X"].copy_(A["Xs"][i % 2])
        if sync:
            torch.cuda.synchronize()
        svdq.quantize_act(bufs["X"], A["inv"], A["L1"], x_codes=bufs["xc"], x_scales=bufs["xs"], T=bufs["T"],
                          workspace_buf=bufs["ws"])
        if sync:
            torch.cuda.synchronize()
        svdq.pack_residual(A["Rs"][i % 3], r_codes=bufs["rc"], r_scales=bufs["rs"])
        if sync:
            torch.cuda.synchronize()
        svdq.linear(bufs["xc"], bufs["xs"], bufs["T"], bufs["rc"], bufs["rs"], A["L2"], A["bias"],
                    A["M"], A["K"], A["N"], Y=bufs["Y"])
        if sync:
            torch.cuda.synchronize()
        outs.append(bufs["Y"].clone())
        # the second layer reads the first layer's output as its X
        svdq.quantize_act(bufs["Y"], B["inv"], B["L1"], x_codes=bufs["xc2"], x_scales=bufs["xs2"], T=bufs["T2"],
                          workspace_buf=bufs["ws"])
        if sync:
            torch.cuda.synchronize()
        svdq.linear(bufs["xc2"], bufs["xs2"], bufs["T2"], B["rc"], B["rs"], B["L2"], None,
                    A["M"], A["N"], B["N"], Y=bufs["Y2"])
        if sync:
            torch.cuda.synchronize()
        outs.append(bufs["Y2"].clone())
    return outs


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_overlapped_launches_keep_stream_order(case):
    import torch
    import bit_w4a4_quantized_smooth_b200 as svdq
    from tests.test_gpu_parity import rel_fro
    name, M, K, N, N2, r = case
    p = prepare(name, 2 * M, K, N, r)          # two activations: rows [0, M) and [M, 2M)
    q = prepare(name, M, N, N2, r)             # the second layer (K = N)
    d = to_device(p)
    e = to_device(q)
    R3 = [d["R"], torch.roll(d["R"], 1, dims=1), -d["R"]]
    A = dict(Xs=[d["X"][:M].contiguous(), d["X"][M:].contiguous()], inv=d["inv"], L1=d["L1"], L2=d["L2"],
             bias=d["bias"], Rs=R3, M=M, K=K, N=N)
    brc, brs = svdq.pack_residual(e["R"])
    B = dict(inv=e["inv"], L1=e["L1"], L2=e["L2"], rc=brc, rs=brs, N=N2)
    xc, xs, T = svdq.quantize_act(A["Xs"][0], A["inv"], A["L1"])
    rc, rs = svdq.pack_residual(d["R"])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=xc.device)
    xc2, xs2, T2 = svdq.quantize_act(Y.zero_(), B["inv"], B["L1"])
    # one workspace for both activation calls (zero-filled; each call leaves its counters at zero)
    ws_bytes = max(svdq.binding.quantize_act_workspace_bytes(M, K, r),
                   svdq.binding.quantize_act_workspace_bytes(M, N, r), 16)
    bufs = dict(X=torch.empty_like(A["Xs"][0]), xc=xc, xs=xs, T=T, rc=rc, rs=rs, Y=Y, xc2=xc2, xs2=xs2, T2=T2,
                Y2=torch.empty((M, N2), dtype=torch.bfloat16, device=xc.device),
                ws=torch.zeros(ws_bytes, dtype=torch.uint8, device=xc.device))
    torch.cuda.synchronize()
    steps = 6
    try:
        svdq.set_launch_overlap(False)
        ref = _sequence(svdq, torch, bufs, A, B, steps, sync=True)
        svdq.set_launch_overlap(True)
        got = _sequence(svdq, torch, bufs, A, B, steps, sync=False)
        torch.cuda.synchronize()
        assert svdq.sync_status()[0] == 0
        for i, (a, b) in enumerate(zip(got, ref)):
            assert torch.equal(a, b), i
        # the same sequence captured into a CUDA graph (programmatic edges)
        side = torch.cuda.Stream(xc.device)
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            _sequence(svdq, torch, bufs, A, B, 1, sync=False)
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            gout = _sequence(svdq, torch, bufs, A, B, 3, sync=False)
        for o in gout:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert svdq.sync_status()[0] == 0
        for i, (a, b) in enumerate(zip(gout, ref[:6])):
            assert torch.equal(a, b), ("graph", i)
        del g
    finally:
        svdq.set_launch_overlap(True)
    # anchor: the first layer's first output against the oracle
    Xa = p.X[:M]
    oxc, oxs, oT = oracle.quantize_act(Xa, p.inv, p.L1, r)
    orc, ors = oracle.pack_residual(p.R)
    rows = np.arange(0, M, 7)
    Yo = oracle.linear_rows(oxc, oxs, oT, orc, ors, p.L2, p.bias, M, K, N, r, rows)
    Yg = bf16_to_np_bits(ref[0])[rows]
    Yg = (Yg.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert rel_fro(Yg, Yo) <= 2e-3
