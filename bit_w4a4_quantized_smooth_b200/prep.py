"""Offline preparation of one layer on the GPU (run once per weight, untimed).

SVDQuant's preparation (chattools.cn article 584, "technical principles";
ai-digest.ru abstract): smoothing factors move activation outliers into the
weights, the SVD of the smoothed weight gives the 16-bit low-rank branch,
and the rest is the residual that the packer quantises to 4 bits.

    lambda_j = sqrt(max_i |X_ij|) / sqrt(max_n |W_jn|)   (1 if either max is 0)
    Wh = diag(lambda) W,  Wh ~ U_r S_r V_r^T  (top-r eigenpairs of the Gram matrix)
    L1 = bf16(U_r S_r), L2 = bf16(V_r^T), R = fp32(Wh - L1 L2)

It uses torch's library linear algebra (matmul, eigh, QR, SVD) in fp64 on the
device: preparation is not part of the forward pass that the library's
kernels run.  lowrank() takes the top-r eigenpairs of the Gram matrix;
lowrank_randomized() a randomized subspace iteration for many layers at once.
"""

from __future__ import annotations

import torch


def smoothing(Xcal: torch.Tensor, W: torch.Tensor):
    """-> (lambda fp32 [K], inv_lambda fp32 [K])."""
    return smoothing_from_stats(Xcal.abs().amax(dim=0).float(), W)


def smoothing_from_stats(x_amax: torch.Tensor, W: torch.Tensor):
    """The smoothing factors from calibration statistics: x_amax fp32 [K],
    the per-channel max |X| over every calibration batch (gathered on the
    device by svdq_channel_absmax, batch by batch).
    -> (lambda fp32 [K], inv_lambda fp32 [K])."""
    a = x_amax.double()
    b = W.abs().amax(dim=1).double()
    lam = torch.where((a == 0) | (b == 0), torch.ones_like(a), a.sqrt() / b.sqrt()).float()
    inv = torch.ones_like(lam) / lam  # fp32 quotient, rounded once
    return lam, inv


def lowrank(W: torch.Tensor, lam: torch.Tensor, r: int):
    """-> (L1 bf16 [K][r] or None, L2 bf16 [r][N] or None, R fp32 [K][N])."""
    Wh = lam.double()[:, None] * W.double()
    K, N = Wh.shape
    if r == 0:
        return None, None, Wh.float()
    if K <= N:
        G = Wh @ Wh.T
        w, Q = torch.linalg.eigh(G)
        U = Q[:, -r:].flip(1)
        s = w[-r:].flip(0).clamp_min(0).sqrt()
        V = (Wh.T @ U) / torch.where(s > 0, s, torch.ones_like(s))
    else:
        G = Wh.T @ Wh
        w, Q = torch.linalg.eigh(G)
        V = Q[:, -r:].flip(1)
        s = w[-r:].flip(0).clamp_min(0).sqrt()
        U = (Wh @ V) / torch.where(s > 0, s, torch.ones_like(s))
    L1 = (U * s).to(torch.bfloat16)
    L2 = V.T.contiguous().to(torch.bfloat16)
    R = (Wh - L1.double() @ L2.double()).float()
    return L1.contiguous(), L2.contiguous(), R.contiguous()


def lowrank_randomized(W: torch.Tensor, lam: torch.Tensor, r: int, oversample: int = 16,
                       power_iters: int = 2, seed: int = 0):
    """The same factors as lowrank() from a randomized range finder instead
    of a full eigendecomposition: Halko, Martinsson and Tropp, "Finding
    structure with randomness" (SIAM Review 53, 2011), Algorithm 4.4
    (randomized subspace iteration, re-orthonormalised after every product),
    then the SVD of the small projected matrix.  fp64 on the device, a few
    matmuls and QRs of width r + oversample: milliseconds where the Gram
    eigendecomposition of a 3072-wide layer takes most of a second.  The
    top-r subspace is approximate (exact on a rank-r matrix); R is still
    exactly Wh - L1 L2 rounded to fp32, so the layer's reconstruction holds.
    -> (L1 bf16 [K][r] or None, L2 bf16 [r][N] or None, R fp32 [K][N])."""
    Wh = lam.double()[:, None] * W.double()
    K, N = Wh.shape
    if r == 0:
        return None, None, Wh.float()
    l = min(r + oversample, K, N)
    gen = torch.Generator(device=Wh.device)
    gen.manual_seed(seed)
    omega = torch.randn((N, l), generator=gen, device=Wh.device, dtype=torch.float64)
    Q, _ = torch.linalg.qr(Wh @ omega)
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(Wh.T @ Q)
        Q, _ = torch.linalg.qr(Wh @ Z)
    Ub, s, Vt = torch.linalg.svd(Q.T @ Wh, full_matrices=False)
    U = Q @ Ub[:, :r]
    L1 = (U * s[:r]).to(torch.bfloat16)
    L2 = Vt[:r].contiguous().to(torch.bfloat16)
    R = (Wh - L1.double() @ L2.double()).float()
    return L1.contiguous(), L2.contiguous(), R.contiguous()


def attach_lora(L1, L2, lam: torch.Tensor, A: torch.Tensor, B: torch.Tensor):
    """Join a LoRA adapter A bf16 [K][ra], B bf16 [ra][N] to the low-rank
    branch without re-quantising the residual (chattools.cn
    "SVDQuant的主要功能", item LoRA集成): with Xh = X diag(lambda)^-1,
    Xh [L1 | diag(lambda) A] [L2 ; B] = Xh L1 L2 + X A B.
    -> (L1' bf16 [K][r+ra], L2' bf16 [r+ra][N]); lambda A is one fp32
    product per element, rounded once to bf16."""
    LA = (lam.float()[:, None] * A.float()).to(torch.bfloat16)
    L1n = LA if L1 is None else torch.cat([L1, LA], dim=1)
    L2n = B if L2 is None else torch.cat([L2, B], dim=0)
    return L1n.contiguous(), L2n.contiguous()


# ------------------------------------------------------- global scales ----
# NVFP4 with a per-tensor global scale g (two-level scaling: a group
# dequantises to q * decode(s) * g).  g is a power of two chosen so that the
# tensor's largest group lands in E4M3's top binade: small groups then keep
# normal (not subnormal or zero) scales, and groups above 6 * 448 no longer
# saturate.  With powers of two the two-level encoding of Z is the plain
# encoding of Z / g, so the library's calls take pre-scaled operands
# (include/svdq.h, svdq_linear_scaled).

E4M3_MAX = 448.0


def global_scale(amax: float) -> float:
    """The power of two 2^ceil(log2(amax / (6 * 448))) (1 for amax = 0)."""
    import math
    amax = float(amax)
    if not (amax > 0.0) or not math.isfinite(amax):
        return 1.0
    m, e = math.frexp(amax / (6.0 * E4M3_MAX))  # amax / 2688 = m 2^e, m in [0.5, 1)
    return math.ldexp(1.0, e if m > 0.5 else e - 1)


def _exact_scale(t: torch.Tensor, f: float, name: str) -> torch.Tensor:
    out = (t.float() * f).to(t.dtype)
    if not torch.equal((out.float() / f).to(t.dtype), t):
        raise ValueError(f"{name}: scaling by {f} is not exact (under- or overflow)")
    return out


def apply_global_scales(inv_lambda: torch.Tensor, L2, R: torch.Tensor, gx: float, gw: float):
    """Operands of the two-level layer for the plain calls:
    -> (inv_lambda / g_x, L2 / g_w or None, R / g_w, alpha = g_x g_w).
    Every product is exact (checked: a power of two that under- or
    overflows raises)."""
    for g in (gx, gw):
        import math
        if not (g > 0.0) or math.frexp(g)[0] != 0.5:
            raise ValueError(f"global scale {g} is not a power of two")
    inv_s = _exact_scale(inv_lambda, 1.0 / gx, "inv_lambda")
    L2_s = None if L2 is None else _exact_scale(L2, 1.0 / gw, "L2")
    R_s = _exact_scale(R, 1.0 / gw, "R")
    return inv_s, L2_s, R_s, gx * gw


def activation_global_scale(x_amax: torch.Tensor, inv_lambda: torch.Tensor) -> float:
    """g_x from calibration statistics: the largest |Xh| = max_k amax_k inv_lambda_k."""
    return global_scale(float((x_amax.float() * inv_lambda.float()).max()))
