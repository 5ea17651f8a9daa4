"""Pins for the product's offline preparation (bit_w4a4_quantized_smooth_b200.prep).

prep.smoothing and prep.lowrank build every layer the benchmark times, on the
device, with torch's library linear algebra.  They are checked here on the
CPU (the same torch calls) against:

* the oracle's smoothing, bit for bit (lambda and its fp32 reciprocal);
* exact reconstruction: L1 L2 + R equals diag(lambda) W to half an fp32 ulp
  of R per element, since R is the fp32 rounding of Wh - L1 L2;
* Eckart-Young-Mirsky (the principles section of the chattools.cn SVDQuant
  article: the SVD removes the dominant singular values): the spectral norm
  of R is sigma_{r+1} of Wh up to the bf16 rounding of the factors, so the
  planted outlier directions of the test weights have left R.
"""

import numpy as np
import pytest

import oracle
from svdq_inputs import bf16_bits_to_f32, make_layer_inputs

torch = pytest.importorskip("torch")


def _t16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _f64(t):
    return t.double().numpy()


CASES = [("tiny", None, None, None, None), ("flux_qkv", 96, 192, 320, 16), ("flux_mlp_down", 64, 256, 128, 32)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_smoothing_matches_oracle_bit_exact(case):
    from bit_w4a4_quantized_smooth_b200 import prep
    name, M, K, N, r = case
    li = make_layer_inputs(name, M=M, K=K, N=N, r=r)
    X = li.Xcal.copy()
    W = li.W.copy()
    X[:, 3] = 0          # a channel the calibration never sees: lambda = 1
    W[5, :] = 0x8000     # an input channel whose weights are all -0: lambda = 1
    lam, inv = prep.smoothing(_t16(X), _t16(W))
    olam, oinv = oracle.smooth(X, W)
    assert np.array_equal(lam.numpy().view(np.uint32), olam.view(np.uint32))
    assert np.array_equal(inv.numpy().view(np.uint32), oinv.view(np.uint32))
    assert lam[3] == 1.0 and lam[5] == 1.0


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_lowrank_reconstructs_smoothed_weight(case):
    from bit_w4a4_quantized_smooth_b200 import prep
    name, M, K, N, r = case
    li = make_layer_inputs(name, M=M, K=K, N=N, r=r)
    lam, _ = prep.smoothing(_t16(li.Xcal), _t16(li.W))
    L1, L2, R = prep.lowrank(_t16(li.W), lam, li.r)
    assert L1.dtype == torch.bfloat16 and L2.dtype == torch.bfloat16 and R.dtype == torch.float32
    assert tuple(L1.shape) == (li.K, li.r) and tuple(L2.shape) == (li.r, li.N)
    Wh = lam.double().numpy()[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)
    P = _f64(L1) @ _f64(L2)
    Rn = R.numpy().astype(np.float64)
    half_ulp = np.spacing(np.abs(R.numpy())).astype(np.float64) / 2
    assert np.all(np.abs(P + Rn - Wh) <= half_ulp * (1 + 1e-9) + 1e-300)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_lowrank_residual_spectral_norm(case):
    """||R||_2 = sigma_{r+1}(Wh) up to the bf16 rounding of L1 and L2
    (at most 2^-8 relative per factor entry, so a perturbation of the
    removed part of about 2^-7 sigma_1); a wrong split, transpose or rank
    leaves sigma_1-sized residue."""
    from bit_w4a4_quantized_smooth_b200 import prep
    name, M, K, N, r = case
    li = make_layer_inputs(name, M=M, K=K, N=N, r=r)
    lam, _ = prep.smoothing(_t16(li.Xcal), _t16(li.W))
    L1, L2, R = prep.lowrank(_t16(li.W), lam, li.r)
    Wh = lam.double().numpy()[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)
    s = np.linalg.svd(Wh, compute_uv=False)
    rn = np.linalg.norm(R.numpy().astype(np.float64), 2)
    assert rn >= s[li.r] * (1 - 1e-6)
    assert rn <= s[li.r] + 2.0 ** -7 * s[0]
    # and the oracle's residual has the same spectral norm to that precision
    olam, _ = oracle.smooth(li.Xcal, li.W)
    _, _, oR, osig = oracle.lowrank(li.W, olam, li.r)
    assert abs(np.linalg.norm(oR.astype(np.float64), 2) - rn) <= 2.0 ** -7 * s[0]
    assert np.allclose(osig[: li.r + 1], s[: li.r + 1], rtol=1e-9)


def test_lowrank_rank_zero_is_the_smoothed_weight():
    from bit_w4a4_quantized_smooth_b200 import prep
    li = make_layer_inputs("flux_qkv", M=32, K=128, N=64, r=0)
    lam, _ = prep.smoothing(_t16(li.Xcal), _t16(li.W))
    L1, L2, R = prep.lowrank(_t16(li.W), lam, 0)
    assert L1 is None and L2 is None
    Wh = (lam.double().numpy()[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)).astype(np.float32)
    assert np.array_equal(R.numpy(), Wh)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_randomized_lowrank_reconstructs_and_captures_the_top_subspace(case):
    """The randomized range finder gives a residual that reconstructs Wh to
    half an fp32 ulp (by construction) and whose spectral norm is within a
    few percent of sigma_{r+1} (Halko et al., Thm. 10.6: with 2 power
    iterations and 16 extra samples the excess is a small multiple of
    sigma_{r+1} for these spectra); missing a planted direction would leave
    sigma_1-sized residue."""
    from bit_w4a4_quantized_smooth_b200 import prep
    name, M, K, N, r = case
    li = make_layer_inputs(name, M=M, K=K, N=N, r=r)
    lam, _ = prep.smoothing(_t16(li.Xcal), _t16(li.W))
    L1, L2, R = prep.lowrank_randomized(_t16(li.W), lam, li.r)
    assert tuple(L1.shape) == (li.K, li.r) and tuple(L2.shape) == (li.r, li.N)
    Wh = lam.double().numpy()[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)
    Rn = R.numpy().astype(np.float64)
    half_ulp = np.spacing(np.abs(R.numpy())).astype(np.float64) / 2
    assert np.all(np.abs(_f64(L1) @ _f64(L2) + Rn - Wh) <= half_ulp * (1 + 1e-9) + 1e-300)
    s = np.linalg.svd(Wh, compute_uv=False)
    rn = np.linalg.norm(Rn, 2)
    assert s[li.r] * (1 - 1e-6) <= rn <= 1.1 * s[li.r] + 2.0 ** -7 * s[0], (rn, s[li.r], s[0])


def test_randomized_lowrank_is_exact_on_exact_rank():
    """A weight of rank exactly r is recovered (residual = the bf16
    rounding of the factors only)."""
    from bit_w4a4_quantized_smooth_b200 import prep
    rng = np.random.default_rng(5)
    K, N, r = 96, 160, 8
    W = torch.from_numpy(rng.standard_normal((K, r)) @ rng.standard_normal((r, N))).to(torch.bfloat16)
    lam = torch.ones(K)
    L1, L2, R = prep.lowrank_randomized(W, lam, r)
    Wd = W.double().numpy()
    assert np.linalg.norm(R.numpy().astype(np.float64), 2) <= 2.0 ** -7 * np.linalg.norm(Wd, 2)
