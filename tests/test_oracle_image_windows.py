"""Pins of the oracle's shifted-window attention over feature maps."""
import numpy as np
import pytest

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


# ------------------------------------------------------------------ backward

def test_backward_finite_differences_shifted():
    """Central differences of L = sum(dO o O) through the oracle's own forward,
    on a 16 x 16 map shifted by 4 (masked windows in the last row and column)."""
    B, Hs, Ws, nh, d, r = 1, 16, 16, 2, 4, 2
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=21)
    rng = np.random.default_rng(5)
    do = rng.standard_normal(q.shape)
    s, shift = 0.45, 4
    grads = oracle.bwd_image_windows(q, k, v, u, w, do, s, 8, shift)
    args = [q, k, v, u, w]

    def loss(a):
        o, _ = oracle.fwd_image_windows(*a, s, 8, shift)
        return float((do * o).sum())

    h = 1e-6
    for t, g in enumerate(grads):
        flat = args[t].reshape(-1)
        for idx in rng.choice(flat.size, size=10, replace=False):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[t].reshape(-1)[idx] += h
            minus[t].reshape(-1)[idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = g.reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (t, idx, fd, an)


def test_backward_unshifted_equals_factored_oracle_on_partitioned_windows():
    """Without a shift: the C oracle's backward on windows cut by reshapes, with
    the shared factors' gradients summed over the windows."""
    B, Hs, Ws, nh, d, r = 2, 16, 8, 2, 8, 4
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=22)
    do = np.random.default_rng(6).standard_normal(q.shape)
    dq, dk, dv, du, dw = oracle.bwd_image_windows(q, k, v, u, w, do, 0.35, 8, 0)

    def part(x):
        c = x.shape[-1]
        x = x.reshape(B, Hs // 8, 8, Ws // 8, 8, nh, c).transpose(0, 1, 3, 5, 2, 4, 6)
        return x.reshape(-1, nh, 64, c)

    nw = B * (Hs // 8) * (Ws // 8)
    ub = np.broadcast_to(u[None], (nw, nh, 64, r)).copy()
    wb = np.broadcast_to(w[None], (nw, nh, 64, r)).copy()
    rq, rk, rv, ru, rw = oracle.bwd(part(q), part(k), part(v), ub, wb, part(do), 0.35)
    for got, want in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(part(got), want, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(du, ru.sum(axis=0), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, rw.sum(axis=0), rtol=1e-10, atol=1e-12)


def test_backward_shift_on_one_window_is_four_region_backwards():
    """An 8 x 8 map shifted by 4: the gradients of each 4 x 4 block are those of
    plain attention inside the block (the C oracle on 16 tokens)."""
    nh, d = 2, 8
    q, k, v, _, _ = _maps(1, 8, 8, nh, d, 0, seed=23)
    do = np.random.default_rng(7).standard_normal(q.shape)
    dq, dk, dv, _, _ = oracle.bwd_image_windows(q, k, v, None, None, do, 0.5, 8, 4)
    for y0 in (0, 4):
        for x0 in (0, 4):
            for h in range(nh):
                sl = (0, slice(y0, y0 + 4), slice(x0, x0 + 4), h)
                blk = [t[sl].reshape(1, 1, 16, d) for t in (q, k, v, do)]
                rq, rk, rv, _, _ = oracle.bwd(blk[0], blk[1], blk[2], None, None, blk[3], 0.5)
                for got, want in ((dq, rq), (dk, rk), (dv, rv)):
                    np.testing.assert_allclose(got[sl].reshape(16, d), want[0, 0], rtol=1e-10,
                                               atol=1e-12)


# Plausible mistakes planted in a copy of the oracle's image-window backward
# (text substitution in its source); the pins above must reject every one.
BWD_MUTANTS = [
    ("mask_dropped", "S = np.where(allowed, S, -np.inf)\n                    E = np.exp",
     "S = S\n                    E = np.exp"),
    ("not_rolled_back", "return back(dQ), back(dK), back(dV), dU, dW",
     "return dQ, dK, dV, dU, dW"),
    ("du_not_summed", "dU[h] += dS @ ww[h]", "dU[h] = dS @ ww[h]"),
    ("d_missing", "dS = P * (dP - Dv)", "dS = P * dP"),
    ("dk_unscaled", "dK[b, ys, xs, h] = scale * (dS.T @ Qw)", "dK[b, ys, xs, h] = dS.T @ Qw"),
    ("dw_wrong_operand", "dW[h] += dS.T @ uu[h]", "dW[h] += dS.T @ ww[h]"),
    ("dv_uses_ds", "dV[b, ys, xs, h] = P.T @ dOw", "dV[b, ys, xs, h] = dS.T @ dOw"),
]


def _planted_bwd(old, new):
    import inspect
    src = inspect.getsource(oracle.bwd_image_windows)
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<planted>", "exec"), ns)
    return ns["bwd_image_windows"]


def _fd_pin_holds(bwd):
    B, Hs, Ws, nh, d, r = 1, 16, 16, 2, 4, 2
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=31)
    rng = np.random.default_rng(8)
    do = rng.standard_normal(q.shape)
    s, shift, h = 0.45, 4, 1e-6
    grads = bwd(q, k, v, u, w, do, s, 8, shift)
    args = [q, k, v, u, w]
    loss = lambda a: float((do * oracle.fwd_image_windows(*a, s, 8, shift)[0]).sum())
    for t, g in enumerate(grads):
        for idx in rng.choice(args[t].size, size=6, replace=False):
            plus, minus = [a.copy() for a in args], [a.copy() for a in args]
            plus[t].reshape(-1)[idx] += h
            minus[t].reshape(-1)[idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            if abs(fd - g.reshape(-1)[idx]) > 1e-6 * max(1.0, abs(fd)):
                return False
    return True


def test_backward_pins_hold_for_the_unmodified_copy():
    assert _fd_pin_holds(_planted_bwd("dS = P * (dP - Dv)", "dS = P * (dP - Dv)"))


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_backward_pins_catch_planted_mistake(name, old, new):
    assert not _fd_pin_holds(_planted_bwd(old, new)), name


# The same for the forward: mistakes planted in a copy of fwd_image_windows
# must fail at least one of the forward pins above.
FWD_MUTANTS = [
    ("mask_dropped", "S = np.where(allowed, S, -np.inf)\n                    m = S.max",
     "S = S\n                    m = S.max"),
    ("rolled_the_wrong_way", "np.roll(x, (-shift, -shift), axis=(1, 2)) for x in (q, k, v)",
     "np.roll(x, (shift, shift), axis=(1, 2)) for x in (q, k, v)"),
    ("not_rolled_back", "return (np.roll(O, (shift, shift), axis=(1, 2)), np.roll(L, (shift, shift), axis=(1, 2)))",
     "return (O, L)"),
    ("bias_transposed", "np.asarray(u, dtype=np.float64)[h] @ np.asarray(w, dtype=np.float64)[h].T",
     "np.asarray(w, dtype=np.float64)[h] @ np.asarray(u, dtype=np.float64)[h].T"),
]


def _planted_fwd(old, new):
    import inspect
    src = inspect.getsource(oracle.fwd_image_windows)
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<planted>", "exec"), ns)
    return ns["fwd_image_windows"]


def _fwd_pins_hold(fwd, monkeypatch):
    monkeypatch.setattr(oracle, "fwd_image_windows", fwd)
    try:
        test_unshifted_equals_factored_oracle_on_partitioned_windows()
        test_shift_on_one_window_splits_it_into_four_regions()
        test_interior_shifted_window_needs_no_mask()
    except AssertionError:
        return False
    return True


def test_forward_pins_hold_for_the_unmodified_copy(monkeypatch):
    assert _fwd_pins_hold(_planted_fwd("m = S.max", "m = S.max"), monkeypatch)


@pytest.mark.parametrize("name,old,new", FWD_MUTANTS, ids=[m[0] for m in FWD_MUTANTS])
def test_forward_pins_catch_planted_mistake(name, old, new, monkeypatch):
    assert not _fwd_pins_hold(_planted_fwd(old, new), monkeypatch), name
