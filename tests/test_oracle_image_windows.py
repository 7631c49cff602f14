"""Pins of the oracle's shifted-window attention over feature maps."""
import numpy as np

import oracle
from rank_biased_window_b200.inputs import make_inputs, to_f64


def _maps(B, Hs, Ws, nh, d, r, seed):
    """Image-layout inputs [B, Hs, Ws, heads, d] and shared factors [heads, 64, r]."""
    x = make_inputs(1, B * Hs * Ws, nh, d, r, seed=seed)
    f = {k: to_f64(v)[0] for k, v in x.items()}
    q, k, v = (f[n].reshape(B, Hs, Ws, nh, d) for n in ("q", "k", "v"))
    u = f["u"][:64].transpose(1, 0, 2) if r else None     # [heads, 64, r]
    w = f["w"][:64].transpose(1, 0, 2) if r else None
    return q, k, v, u, w


def test_unshifted_equals_factored_oracle_on_partitioned_windows():
    B, Hs, Ws, nh, d, r = 2, 16, 24, 3, 8, 4
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=11)
    o, lse = oracle.fwd_image_windows(q, k, v, u, w, 0.3, 8, 0)

    def part(x):  # [B, Hs, Ws, nh, c] -> [B * nWin, nh, 64, c] by reshapes only
        c = x.shape[-1]
        x = x.reshape(B, Hs // 8, 8, Ws // 8, 8, nh, c).transpose(0, 1, 3, 5, 2, 4, 6)
        return x.reshape(-1, nh, 64, c)

    nw = B * (Hs // 8) * (Ws // 8)
    ub = np.broadcast_to(u[None], (nw, nh, 64, r)).copy()
    wb = np.broadcast_to(w[None], (nw, nh, 64, r)).copy()
    ro, rl = oracle.fwd(part(q), part(k), part(v), ub, wb, 0.3)
    np.testing.assert_allclose(part(o), ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(part(lse[..., None])[..., 0], rl, rtol=1e-12, atol=1e-12)


def test_shift_on_one_window_splits_it_into_four_regions():
    """An 8 x 8 map shifted by 4 is one window holding four 4 x 4 regions that
    were not neighbours: each attends only within itself."""
    B, nh, d = 1, 2, 8
    q, k, v, _, _ = _maps(B, 8, 8, nh, d, 0, seed=12)
    o, lse = oracle.fwd_image_windows(q, k, v, None, None, 0.5, 8, 4)
    for y0 in (0, 4):
        for x0 in (0, 4):
            for h in range(nh):
                sl = (0, slice(y0, y0 + 4), slice(x0, x0 + 4), h)
                Q, K, V = (t[sl].reshape(16, d) for t in (q, k, v))
                S = 0.5 * Q @ K.T
                P = np.exp(S - S.max(1, keepdims=True))
                want = (P @ V) / P.sum(1, keepdims=True)
                np.testing.assert_allclose(o[sl].reshape(16, d), want, rtol=1e-12, atol=1e-12)
                lw = S.max(1) + np.log(np.exp(S - S.max(1, keepdims=True)).sum(1))
                np.testing.assert_allclose(lse[sl].reshape(16), lw, rtol=1e-12, atol=1e-12)


def test_interior_shifted_window_needs_no_mask():
    """On a 24 x 24 map shifted by 4, the centre window of the rolled map holds
    original rows and columns 12..19, all neighbours: plain attention."""
    B, nh, d, r = 1, 1, 8, 4
    q, k, v, u, w = _maps(B, 24, 24, nh, d, r, seed=13)
    o, _ = oracle.fwd_image_windows(q, k, v, u, w, 0.4, 8, 4)
    Q, K, V = (t[0, 12:20, 12:20, 0].reshape(64, d) for t in (q, k, v))
    S = 0.4 * Q @ K.T + u[0] @ w[0].T
    P = np.exp(S - S.max(1, keepdims=True))
    want = (P @ V) / P.sum(1, keepdims=True)
    np.testing.assert_allclose(o[0, 12:20, 12:20, 0].reshape(64, d), want, rtol=1e-12, atol=1e-12)
