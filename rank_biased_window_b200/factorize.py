"""Low-rank factors of a materialised bias: the step before the attention path
that turns a dense per-head bias matrix (for example a relative-position table
expanded over a window) into the factors U, W the kernels take, following the
low-rank view of "FlashBias: Fast Computation of Attention with Bias"
(Abstract: a low-rank bias keeps attention fast).

Randomised subspace iteration (Halko, Martinsson and Tropp, "Finding structure
with randomness", 2011: range finder with power iterations, then an SVD of the
small projected matrix):

    Y = B G  (G Gaussian N x (r + p));  repeat q times: Y = B (B^T Y), orthonormalised
    Q = orth(Y);  C^T = B^T Q  (N x (r + p));  C = X S Z^T  (small SVD)
    U = Q X[:, :r] sqrt(S[:r]),  W = Z[:, :r] sqrt(S[:r])

Every product with the N x N bias runs in the library's kernel
(rfb_bias_project, fp32); the QR and SVD of the thin N x (r + p) matrices and
the small products with them are library routines (torch on the bias's
device).  This runs once per model, off the attention path.
"""
from __future__ import annotations

import torch


def _factorize(bias: torch.Tensor, r: int, project, *, oversample: int = 8, power_iters: int = 2,
               seed: int = 0, out_dtype=torch.bfloat16):
    """The algorithm, with project(B, X, transpose) computing B X or B^T X for
    B [H, N, N] and X [H, N, k] (fp32)."""
    if bias.dim() != 3 or bias.shape[1] != bias.shape[2]:
        raise ValueError("bias must be [H, N, N]")
    H, N, _ = bias.shape
    if not (0 < r <= N):
        raise ValueError("need 0 < r <= N")
    k = min(N, r + oversample)
    B = bias.float().contiguous()
    g = torch.Generator(device=B.device)
    g.manual_seed(int(seed))
    G = torch.randn((H, N, k), generator=g, device=B.device, dtype=torch.float32)
    Q, _ = torch.linalg.qr(project(B, G, False))
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(project(B, Q.contiguous(), True))
        Q, _ = torch.linalg.qr(project(B, Z.contiguous(), False))
    Ct = project(B, Q.contiguous(), True)                    # [H, N, k] = (Q^T B)^T
    X, S, Zt = torch.linalg.svd(Ct.transpose(1, 2), full_matrices=False)   # C = X diag(S) Zt
    root = S[:, :r].clamp_min(0).sqrt()
    U = torch.bmm(Q, X[:, :, :r]) * root[:, None, :]
    W = Zt[:, :r, :].transpose(1, 2) * root[:, None, :]
    U, W = U.to(out_dtype).contiguous(), W.to(out_dtype).contiguous()
    # reported error of the rounded factors (a library product: diagnostics only)
    R = B - torch.bmm(U.float(), W.float().transpose(1, 2))
    rel = torch.linalg.matrix_norm(R) / torch.linalg.matrix_norm(B).clamp_min(1e-30)
    return U, W, rel


def factorize_bias(bias: torch.Tensor, r: int, *, oversample: int = 8, power_iters: int = 2,
                   seed: int = 0, out_dtype=torch.bfloat16):
    """bias ``[H, N, N]`` on a CUDA device (any float dtype).  Returns
    ``(U, W, rel_err)``: U, W ``[H, N, r]`` in ``out_dtype`` and the relative
    Frobenius error ``||B - U W^T|| / ||B||`` per head, measured in fp32 on the
    rounded factors.  r + oversample (capped at N) must be at most 80."""
    from .binding import bias_project
    if not bias.is_cuda:
        raise ValueError("factorize_bias runs its products on the GPU: bias must be a CUDA tensor")
    return _factorize(bias, r, lambda B, X, t: bias_project(B, X, t), oversample=oversample,
                      power_iters=power_iters, seed=seed, out_dtype=out_dtype)


def relative_position_bias(H: int, wh: int, ww: int, *, seed: int = 0, device="cpu"):
    """Synthetic relative-position bias for wh x ww windows, [H, N, N] with
    N = wh * ww: per head a random mixture of a Gaussian bump, two cosine
    ridges and a smoothed random table in (dy, dx), evaluated at every
    query-key offset.  A stand-in for a trained relative-position table (no
    trained weights are used)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    ys = torch.arange(wh).repeat_interleave(ww)
    xs = torch.arange(ww).repeat(wh)
    dy = (ys[:, None] - ys[None, :]).float()
    dx = (xs[:, None] - xs[None, :]).float()
    out = torch.empty((H, wh * ww, wh * ww))
    iy = (dy + wh - 1).long()
    ix = (dx + ww - 1).long()
    for h in range(H):
        a, b, c = torch.randn(3, generator=g).tolist()
        sy, sx = (0.2 + torch.rand(2, generator=g) * 0.5).tolist()
        fy, fx = (torch.rand(2, generator=g) * 0.6).tolist()
        # plus a random table over the (2 wh - 1) x (2 ww - 1) offsets, smoothed
        # by a 3 x 3 box filter (rougher, slower-decaying spectrum)
        t = torch.randn((1, 1, 2 * wh - 1, 2 * ww - 1), generator=g)
        t = torch.nn.functional.avg_pool2d(torch.nn.functional.pad(t, (1, 1, 1, 1), mode="replicate"),
                                           3, stride=1)[0, 0]
        out[h] = (a * torch.exp(-(dy * sy) ** 2 / 8 - (dx * sx) ** 2 / 8)
                  + b * torch.cos(fy * dy) + c * torch.cos(fx * dx) + 0.5 * t[iy, ix])
    return out.to(device)
