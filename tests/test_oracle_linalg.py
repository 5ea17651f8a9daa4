"""Pins for the oracle's offline preparation: smoothing, top-r SVD, residual.

Checked against numpy.linalg (an independent library), the Eckart-Young-Mirsky
theorem (SVDQuant relies on it to remove the dominant singular values: the
principles section of the chattools.cn SVDQuant article), exact
reconstruction and the closed form of alpha = 0.5 smoothing.
"""

import numpy as np
import pytest

from svdq_inputs import bf16_bits_from_f64, bf16_bits_to_f32, make_layer_inputs


def _spread_matrix(K, N, seed, decay=0.9):
    """Random K x N matrix with well separated singular values."""
    rng = np.random.default_rng(seed)
    u, _ = np.linalg.qr(rng.standard_normal((K, min(K, N))))
    v, _ = np.linalg.qr(rng.standard_normal((N, min(K, N))))
    s = 5.0 * decay ** np.arange(min(K, N))
    return (u * s) @ v.T, s


def test_sym_eig_top_matches_numpy(oracle_lib):
    rng = np.random.default_rng(11)
    for n in (1, 2, 3, 17, 60):
        B = rng.standard_normal((n, n))
        A = B + B.T
        k = min(n, 6)
        vals, vecs = oracle_lib.sym_eig_top(A, k)
        w, V = np.linalg.eigh(A)
        ref = w[::-1][:k]
        scale = max(1.0, np.max(np.abs(w)))
        assert np.allclose(vals, ref, rtol=0, atol=1e-12 * scale)
        for j in range(k):
            r = A @ vecs[:, j] - vals[j] * vecs[:, j]
            assert np.linalg.norm(r) <= 1e-10 * scale
        assert np.allclose(vecs.T @ vecs, np.eye(k), atol=1e-10)


@pytest.mark.parametrize("K,N", [(40, 70), (70, 40), (33, 33)])
def test_svd_top_matches_numpy(oracle_lib, K, N):
    A, s_true = _spread_matrix(K, N, seed=K * 100 + N)
    r = 8
    U, s, V = oracle_lib.svd_top(A, r)
    s_np = np.linalg.svd(A, compute_uv=False)
    assert np.allclose(s, s_np[: r + 1], rtol=1e-12, atol=1e-12 * s_np[0])
    Un, _, Vt = np.linalg.svd(A)
    for j in range(r):  # singular vectors up to sign (gaps are 10 %)
        assert abs(abs(U[:, j] @ Un[:, j]) - 1) < 1e-9
        assert abs(abs(V[:, j] @ Vt[j]) - 1) < 1e-9


@pytest.mark.parametrize("K,N,r", [(48, 80, 5), (80, 48, 12), (64, 64, 1)])
def test_eckart_young_mirsky(oracle_lib, K, N, r):
    """||A - U_r S_r V_r^T||_2 = sigma_{r+1}, ||.||_F^2 = sum_{i>r} sigma_i^2."""
    A, _ = _spread_matrix(K, N, seed=r + K)
    U, s, V = oracle_lib.svd_top(A, r)
    E = A - (U * s[:r]) @ V.T
    s_all = np.linalg.svd(A, compute_uv=False)
    assert abs(np.linalg.norm(E, 2) - s[r]) <= 1e-9 * s[r]
    assert abs(np.linalg.norm(E) ** 2 - np.sum(s_all[r:] ** 2)) <= 1e-9 * np.sum(s_all[r:] ** 2)


def test_planted_rank_is_recovered(oracle_lib):
    """The tiny workload's planted rank-4 term dominates: the top 4 singular
    values of diag(lambda) W agree with numpy's, and sigma_5 drops sharply."""
    li = make_layer_inputs("tiny", M=64, K=256, N=192, r=8)
    lam, _ = oracle_lib.smooth(li.Xcal, li.W)
    Wh = lam.astype(np.float64)[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)
    U, s, V = oracle_lib.svd_top(Wh, 8)
    s_np = np.linalg.svd(Wh, compute_uv=False)
    assert np.allclose(s, s_np[:9], rtol=1e-10)
    assert s[3] > 3 * s[4]


def test_lowrank_reconstruction(oracle_lib):
    """L1 L2 + R = diag(lambda) W up to the fp32 rounding of R (bf16 factors)."""
    li = make_layer_inputs("tiny", M=64, K=128, N=96, r=16)
    lam, _ = oracle_lib.smooth(li.Xcal, li.W)
    L1, L2, R, s = oracle_lib.lowrank(li.W, lam, 16)
    Wh = lam.astype(np.float64)[:, None] * bf16_bits_to_f32(li.W).astype(np.float64)
    L1d = bf16_bits_to_f32(L1).astype(np.float64)
    L2d = bf16_bits_to_f32(L2).astype(np.float64)
    recon = L1d @ L2d + R.astype(np.float64)
    ulp = np.spacing(np.abs(R)).astype(np.float64)
    assert np.all(np.abs(recon - Wh) <= 0.5 * ulp + 1e-14 * np.abs(Wh).max())
    # the fp64 factors (before bf16 rounding) reconstruct the EYM residual
    U, s2, V = oracle_lib.svd_top(Wh, 16)
    assert np.allclose(s, s2)
    assert np.linalg.norm(Wh - (U * s2[:16]) @ V.T, 2) == pytest.approx(s2[16], rel=1e-8)


def test_lowrank_exact_rank(oracle_lib):
    """W of exact rank <= r leaves only the bf16-factor residue in R."""
    rng = np.random.default_rng(3)
    K, N, q = 96, 64, 3
    # small-integer outer products: every entry is an integer <= 27, exact in bf16
    Wf = rng.integers(-3, 4, (K, q)).astype(np.float64) @ rng.integers(-3, 4, (q, N))
    W = bf16_bits_from_f64(Wf)
    assert np.array_equal(bf16_bits_to_f32(W).astype(np.float64), Wf)
    lam = np.ones(K, dtype=np.float32)
    L1, L2, R, s = oracle_lib.lowrank(W, lam, 4)
    # sigma_4 of an exact rank-3 matrix: the Gram-matrix route resolves a zero
    # singular value only to sqrt(eps) * sigma_1 (the eigenvalue itself is
    # exact to eps * sigma_1^2)
    assert s[3] < 1e-7 * s[0]
    # R is only the residue of rounding the factors to bf16 (8 significant bits)
    assert np.abs(R).max() < 2.0 ** -6 * np.abs(Wf).max()
    U, s64, V = oracle_lib.svd_top(Wf, 3)
    assert np.abs(Wf - (U * s64[:3]) @ V.T).max() < 1e-12 * np.abs(Wf).max()


def test_lowrank_rank_zero(oracle_lib):
    li = make_layer_inputs("tiny", M=32, K=64, N=48, r=0)
    lam, _ = oracle_lib.smooth(li.Xcal, li.W)
    L1, L2, R, s = oracle_lib.lowrank(li.W, lam, 0)
    Wh = (lam.astype(np.float64)[:, None] * bf16_bits_to_f32(li.W)).astype(np.float32)
    assert np.array_equal(R, Wh)


def test_smoothing_max_equalisation(oracle_lib):
    """alpha = 0.5: max_i |Xh_ij| = max_n |Wh_jn| = sqrt(a_j b_j)."""
    li = make_layer_inputs("tiny", M=128, K=256, N=64)
    lam, inv = oracle_lib.smooth(li.Xcal, li.W)
    X = bf16_bits_to_f32(li.X).astype(np.float64)
    W = bf16_bits_to_f32(li.W).astype(np.float64)
    a = np.abs(X).max(0)
    b = np.abs(W).max(1)
    closed = np.sqrt(a * b)
    xh = np.abs(X / lam.astype(np.float64)).max(0)
    wh = np.abs(W * lam.astype(np.float64)[:, None]).max(1)
    assert np.allclose(xh, closed, rtol=1e-6)
    assert np.allclose(wh, closed, rtol=1e-6)
    # outlier channels are the ones with the largest smoothing factors
    assert np.argmax(lam) in np.argsort(a)[-8:]


def test_smoothing_identity(oracle_lib):
    """Xh Wh = X W: exactly (to fp64 rounding) with X / lambda, and within
    the fp32 rounding of inv_lambda and of the product for X * inv_lambda."""
    li = make_layer_inputs("tiny", M=32, K=128, N=48)
    lam, inv = oracle_lib.smooth(li.Xcal, li.W)
    X = bf16_bits_to_f32(li.X).astype(np.float64)
    W = bf16_bits_to_f32(li.W).astype(np.float64)
    l64 = lam.astype(np.float64)
    ref = X @ W
    got = (X / l64) @ (W * l64[:, None])
    assert np.linalg.norm(got - ref) <= 1e-12 * np.linalg.norm(ref)
    xh32 = (bf16_bits_to_f32(li.X) * inv[None, :]).astype(np.float64)  # numpy fp32 product
    got32 = xh32 @ (W * l64[:, None])
    assert np.linalg.norm(got32 - ref) <= 3e-7 * np.linalg.norm(ref)


def test_smoothing_zero_channel(oracle_lib):
    X = np.zeros((4, 64), dtype=np.uint16)
    W = bf16_bits_from_f64(np.ones((64, 8)))
    lam, inv = oracle_lib.smooth(X, W)
    assert np.all(lam == 1.0) and np.all(inv == 1.0)
