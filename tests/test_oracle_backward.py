"""Pins for the fp64 oracle's backward pass (CPU only).

The backward is pinned against torch autograd in fp64 through SDPA with a
float bias mask (library special case), against autograd through plain
attention over the concatenated operands [sQ | U], [K | W] (the identity of the
"Rank-Factorized Implicit Neural Bias" abstract), against central finite
differences, and against identities the chain rule fixes.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from rank_biased_window_b200.inputs import make_inputs, to_f64


def _rand(B, H, N, d, r, seed):
    t = make_inputs(B, H, N, d, r, seed, with_dout=True)
    return {k: to_f64(v) for k, v in t.items()}


def _autograd_mask(x, s, r):
    t = {k: torch.from_numpy(v.copy()).requires_grad_(True) for k, v in x.items() if k != "dout"}
    mask = t["u"] @ t["w"].transpose(-1, -2) if r else None
    o = F.scaled_dot_product_attention(t["q"], t["k"], t["v"], attn_mask=mask, scale=s)
    o.backward(torch.from_numpy(x["dout"]))
    g = {k: t[k].grad.numpy() for k in ("q", "k", "v")}
    if r:
        g["u"], g["w"] = t["u"].grad.numpy(), t["w"].grad.numpy()
    return g


@pytest.mark.parametrize("shape", [(1, 1, 1, 4, 2), (1, 2, 9, 8, 4), (2, 1, 33, 16, 8),
                                   (1, 1, 64, 32, 8), (1, 2, 17, 8, 0)])
def test_matches_autograd_through_sdpa(oracle_mod, shape):
    B, H, N, d, r = shape
    x = _rand(B, H, N, d, r, seed=300 + N)
    s = 1.0 / math.sqrt(d)
    dq, dk, dv, du, dw = oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"] if r else None,
                                        x["w"] if r else None, x["dout"], s)
    g = _autograd_mask(x, s, r)
    for name, got in (("q", dq), ("k", dk), ("v", dv), ("u", du), ("w", dw)):
        if got is None:
            assert r == 0
            continue
        np.testing.assert_allclose(got, g[name], rtol=0, atol=1e-11, err_msg=name)


def test_matches_autograd_through_concatenation(oracle_mod):
    """Plain attention over qc = [sQ | U], kc = [K | W] (scale 1): dQ = s dqc[:, :d],
    dU = dqc[:, d:], dK = dkc[:, :d], dW = dkc[:, d:]."""
    B, H, N, d, r = 1, 2, 21, 8, 4
    x = _rand(B, H, N, d, r, seed=77)
    s = 0.3
    dq, dk, dv, du, dw = oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"], x["w"], x["dout"], s)
    q = torch.from_numpy(x["q"]).requires_grad_(True)
    u = torch.from_numpy(x["u"]).requires_grad_(True)
    k = torch.from_numpy(x["k"]).requires_grad_(True)
    w = torch.from_numpy(x["w"]).requires_grad_(True)
    v = torch.from_numpy(x["v"]).requires_grad_(True)
    qc = torch.cat([s * q, u], dim=-1)
    kc = torch.cat([k, w], dim=-1)
    o = F.scaled_dot_product_attention(qc, kc, v, scale=1.0)
    o.backward(torch.from_numpy(x["dout"]))
    for got, ref in ((dq, q.grad), (du, u.grad), (dk, k.grad), (dw, w.grad), (dv, v.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_finite_differences(oracle_mod):
    """Central differences of L = sum(dO * O) w.r.t. every input element."""
    B, H, N, d, r = 1, 1, 8, 4, 2
    x = _rand(B, H, N, d, r, seed=13)
    s = 0.45
    grads = dict(zip("qkvuw", oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"], x["w"],
                                              x["dout"], s)))
    h = 1e-6

    def loss(y):
        o, _ = oracle_mod.fwd(y["q"], y["k"], y["v"], y["u"], y["w"], s)
        return float(np.sum(x["dout"] * o))

    for name in "qkvuw":
        fd = np.zeros_like(x[name])
        flat = fd.reshape(-1)
        for idx in range(flat.size):
            y = {k: v.copy() for k, v in x.items()}
            y[name].reshape(-1)[idx] += h
            lp = loss(y)
            y[name].reshape(-1)[idx] -= 2 * h
            lm = loss(y)
            flat[idx] = (lp - lm) / (2 * h)
        g = grads[name]
        rel = np.linalg.norm(g - fd) / max(np.linalg.norm(fd), 1e-30)
        assert rel < 1e-6, (name, rel)


def test_chain_rule_identities(oracle_mod):
    B, H, N, d, r = 2, 2, 27, 8, 4
    x = _rand(B, H, N, d, r, seed=19)
    s = 0.35
    # A constant column c of W: dU[:, c] = w_c * sum_j dS_ij = 0 (rows of dS sum to 0).
    w = x["w"].copy()
    w[..., 1] = 0.8125
    (dq, dk, dv, du, dw), D = oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"], w, x["dout"], s,
                                             return_D=True)
    assert np.max(np.abs(du[..., 1])) < 1e-13
    # sum_j dV_j = sum_i dO_i (rows of P sum to 1).
    np.testing.assert_allclose(dv.sum(axis=2), x["dout"].sum(axis=2), rtol=0, atol=1e-12)
    # D_i = sum_j P_ij dP_ij equals dO_i . O_i.
    o, _ = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], w, s)
    np.testing.assert_allclose(D, np.sum(x["dout"] * o, axis=-1), rtol=0, atol=1e-12)
    # sum_j dK_j = s * sum_i (sum_j dS_ij) Q_i = 0 because each row of dS sums to
    # zero; likewise sum_j dW_j = 0.
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dw.sum(axis=2), 0.0, atol=1e-12)


def test_query_rows_match_full(oracle_mod):
    B, H, N, d, r = 1, 3, 40, 8, 8
    x = _rand(B, H, N, d, r, seed=23)
    s = 0.3
    (dq, dk, dv, du, dw), D = oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"], x["w"],
                                             x["dout"], s, return_D=True)
    rows = [0, 39, 5, 17]
    q1, u1, d1 = oracle_mod.bwd_query_rows(x["q"], x["k"], x["v"], x["u"], x["w"], x["dout"],
                                           s, 2, rows)
    np.testing.assert_allclose(q1, dq[0, 2][rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(u1, du[0, 2][rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(d1, D[0, 2][rows], rtol=0, atol=1e-14)
    sub = oracle_mod.bwd(x["q"], x["k"], x["v"], x["u"], x["w"], x["dout"], s, bh_range=(1, 3))
    for full, part in zip((dq, dk, dv, du, dw), sub):
        np.testing.assert_array_equal(part, full.reshape(3, N, -1)[1:3])
