"""The .svdq prepared-layer file: exact round trip, and damaged files refused."""

import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bit_w4a4_quantized_smooth_b200 import layer_file


def _layer(K=256, N=144, r=32, bias=True, seed=0):
    g = torch.Generator().manual_seed(seed)
    lam = torch.rand(K, generator=g) + 0.5
    inv = 1.0 / lam
    L1 = torch.randn(K, r, generator=g).to(torch.bfloat16) if r else None
    L2 = torch.randn(r, N, generator=g).to(torch.bfloat16) if r else None
    rc = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    rs = torch.randint(0, 256, (((N + 127) // 128) * 128 * (K // 16),), generator=g, dtype=torch.uint8)
    b = torch.randn(N, generator=g).to(torch.bfloat16) if bias else None
    return dict(lam=lam, inv=inv, L1=L1, L2=L2, rc=rc, rs=rs, bias=b)


@pytest.mark.parametrize("r,bias", [(32, True), (0, False), (128, False)])
def test_round_trip_is_exact(tmp_path, r, bias):
    d = _layer(r=r, bias=bias)
    p = str(tmp_path / "layer.svdq")
    layer_file.save_layer(p, **d)
    back = layer_file.load_layer(p)
    assert (back["K"], back["N"], back["r"]) == (256, 144, r)
    for k, v in d.items():
        if v is None:
            assert back[k] is None, k
        else:
            assert back[k].dtype == v.dtype and torch.equal(back[k], v), k
    assert os.path.getsize(p) % 4 == 0


def test_damaged_files_are_refused(tmp_path):
    d = _layer()
    p = str(tmp_path / "layer.svdq")
    layer_file.save_layer(p, **d)
    blob = open(p, "rb").read()
    bad = tmp_path / "bad.svdq"
    for damaged in (blob[:-9] + blob[-8:],                          # a byte missing
                    blob[:100] + bytes([blob[100] ^ 1]) + blob[101:],  # a flipped bit
                    b"NOTSVDQ!" + blob[8:],                          # wrong magic
                    blob[:40]):                                      # truncated
        bad.write_bytes(damaged)
        with pytest.raises(ValueError):
            layer_file.load_layer(str(bad))


def test_save_checks_the_layouts(tmp_path):
    d = _layer()
    d["rs"] = d["rs"][:-16]
    with pytest.raises(ValueError):
        layer_file.save_layer(str(tmp_path / "x.svdq"), **d)
    d = _layer()
    d["L1"] = d["L1"].float()
    with pytest.raises(ValueError):
        layer_file.save_layer(str(tmp_path / "x.svdq"), **d)


@pytest.mark.gpu
def test_loaded_layer_gives_the_same_output(tmp_path):
    import bit_w4a4_quantized_smooth_b200 as svdq
    from bit_w4a4_quantized_smooth_b200 import prep
    from svdq_inputs import make_layer_inputs
    dev = torch.device("cuda", 0)
    li = make_layer_inputs("flux_qkv", M=200, K=512, N=272)
    X = torch.from_numpy(li.X.view(np.int16)).view(torch.bfloat16).to(dev)
    W = torch.from_numpy(li.W.view(np.int16)).view(torch.bfloat16).to(dev)
    bias = torch.from_numpy(li.bias.view(np.int16)).view(torch.bfloat16).to(dev)
    lam, inv = prep.smoothing(X, W)
    L1, L2, R = prep.lowrank(W, lam, 32)
    rc, rs = svdq.pack_residual(R)
    p = str(tmp_path / "layer.svdq")
    layer_file.save_layer(p, lam, inv, L1, L2, rc, rs, bias)
    ld = layer_file.load_layer(p, dev)
    xc, xs, T = svdq.quantize_act(X, inv, L1)
    Y1 = svdq.linear(xc, xs, T, rc, rs, L2, bias, li.M, li.K, li.N)
    xc2, xs2, T2 = svdq.quantize_act(X, ld["inv"], ld["L1"])
    Y2 = svdq.linear(xc2, xs2, T2, ld["rc"], ld["rs"], ld["L2"], ld["bias"], li.M, ld["K"], ld["N"])
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
