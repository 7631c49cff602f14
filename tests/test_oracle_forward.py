"""Pins for the fp64 oracle's forward pass (CPU only).

Each test checks the oracle against something other than itself: a library
routine (torch SDPA in fp64), brute force with math.fsum, a closed form worked
out by hand, or an invariant that the mathematics fixes.  Together they catch a
dropped bias term, a wrong sign, a transposed factor (W U^T for U W^T), a scale
applied to the bias, a wrong LSE base, and row/column index mix-ups.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from rank_biased_window_b200.inputs import make_inputs, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(B, H, N, d, r, seed):
    t = make_inputs(B, H, N, d, r, seed)
    return {k: to_f64(v) for k, v in t.items()}


def _sdpa(q, k, v, mask, s):
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=s).numpy()


SHAPES = [(1, 1, 1, 4, 0), (1, 2, 7, 8, 0), (2, 3, 33, 16, 0), (1, 1, 64, 32, 0),
          (2, 2, 19, 8, 2), (1, 3, 64, 32, 8), (1, 1, 130, 16, 16), (2, 1, 5, 4, 3)]


@pytest.mark.parametrize("shape", SHAPES)
def test_matches_sdpa_with_bias_mask(oracle_mod, shape):
    """Library special case: SDPA with a float attn_mask adds the mask to the
    scaled scores, which is the bias placement of the FlashBias abstract."""
    B, H, N, d, r = shape
    x = _rand(B, H, N, d, r, seed=100 + N)
    s = 1.0 / math.sqrt(d)
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"] if r else None,
                            x["w"] if r else None, s)
    mask = (x["u"] @ np.swapaxes(x["w"], -1, -2)) if r else None
    ref = _sdpa(x["q"], x["k"], x["v"], mask, s)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    # LSE: natural-log logsumexp of the biased scores (torch.logsumexp).
    sc = torch.from_numpy(x["q"]) @ torch.from_numpy(x["k"]).transpose(-1, -2) * s
    if r:
        sc = sc + torch.from_numpy(mask)
    np.testing.assert_allclose(lse, torch.logsumexp(sc, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_scale_not_applied_to_bias(oracle_mod):
    """s multiplies Q K^T only.  With Q = 0 the scores are the bias alone, so the
    output must not change with s."""
    x = _rand(1, 2, 16, 8, 4, seed=7)
    q0 = np.zeros_like(x["q"])
    o1, l1 = oracle_mod.fwd(q0, x["k"], x["v"], x["u"], x["w"], 0.1)
    o2, l2 = oracle_mod.fwd(q0, x["k"], x["v"], x["u"], x["w"], 3.0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("shape", [(1, 1, 9, 8, 2), (2, 2, 40, 16, 8), (1, 1, 64, 32, 8)])
def test_concatenation_identity(oracle_mod, shape):
    """"Rank-Factorized Implicit Neural Bias", Abstract: concatenating the bias
    factors with the content channels turns the bias addition into one dot
    product.  Plain attention (scale 1, torch SDPA) over [sQ | U] and [K | W]
    must equal the oracle's biased attention."""
    B, H, N, d, r = shape
    x = _rand(B, H, N, d, r, seed=11 + d)
    s = 1.0 / math.sqrt(d)
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], s)
    qc = np.concatenate([s * x["q"], x["u"]], axis=-1)
    kc = np.concatenate([x["k"], x["w"]], axis=-1)
    oc = _sdpa(qc, kc, x["v"], None, 1.0)
    lsec = torch.logsumexp(torch.from_numpy(qc) @ torch.from_numpy(kc).transpose(-1, -2),
                           dim=-1).numpy()
    np.testing.assert_allclose(o, oc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lsec, rtol=0, atol=1e-13)
    # and the score identity itself, elementwise
    lhs = qc @ np.swapaxes(kc, -1, -2)
    rhs = s * (x["q"] @ np.swapaxes(x["k"], -1, -2)) + x["u"] @ np.swapaxes(x["w"], -1, -2)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-13, atol=1e-13)


def test_row_constant_bias(oracle_mod):
    """A bias constant along each row (all W_j equal) cancels in the softmax:
    O equals the unbiased output and LSE_i shifts by exactly U_i . w."""
    x = _rand(2, 2, 24, 8, 4, seed=3)
    wrow = x["w"][:, :, :1, :]
    wconst = np.broadcast_to(wrow, x["w"].shape).copy()
    s = 0.35
    o_b, l_b = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], wconst, s)
    o_0, l_0 = oracle_mod.fwd(x["q"], x["k"], x["v"], None, None, s)
    np.testing.assert_allclose(o_b, o_0, rtol=0, atol=1e-13)
    shift = np.einsum("bhnr,bhr->bhn", x["u"], wrow[:, :, 0, :])
    np.testing.assert_allclose(l_b - l_0, shift, rtol=0, atol=1e-12)


def test_identical_value_rows(oracle_mod):
    """If every V_j equals v, every output row equals v (the rows of P sum to 1)."""
    x = _rand(1, 3, 50, 16, 8, seed=5)
    v = np.broadcast_to(x["v"][:, :, :1, :], x["v"].shape).copy()
    o, _ = oracle_mod.fwd(x["q"], x["k"], v, x["u"], x["w"], 0.25)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)


def test_permutations(oracle_mod):
    """Permuting keys jointly (K, V, W rows) leaves O and LSE unchanged;
    permuting queries jointly (Q, U rows) permutes O and LSE the same way."""
    x = _rand(1, 2, 31, 8, 4, seed=9)
    s = 0.3
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], s)
    rng = np.random.default_rng(0)
    pk = rng.permutation(31)
    o2, l2 = oracle_mod.fwd(x["q"], x["k"][:, :, pk], x["v"][:, :, pk], x["u"],
                            x["w"][:, :, pk], s)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-13)
    pq = rng.permutation(31)
    o3, l3 = oracle_mod.fwd(x["q"][:, :, pq], x["k"], x["v"], x["u"][:, :, pq], x["w"], s)
    np.testing.assert_allclose(o3, o[:, :, pq], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l3, lse[:, :, pq], rtol=0, atol=1e-13)


def _brute(q, k, v, u, w, s):
    """Pure-Python, element by element, exactly rounded sums (math.fsum)."""
    N, d = len(q), len(q[0])
    r = len(u[0]) if u is not None else 0
    O, L = [], []
    for i in range(N):
        sc = []
        for j in range(N):
            bias = math.fsum(u[i][c] * w[j][c] for c in range(r)) if r else 0.0
            sc.append(s * math.fsum(q[i][c] * k[j][c] for c in range(d)) + bias)
        m = max(sc)
        e = [math.exp(t - m) for t in sc]
        z = math.fsum(e)
        O.append([math.fsum(e[j] * v[j][c] for j in range(N)) / z for c in range(d)])
        L.append(m + math.log(z))
    return O, L


@pytest.mark.parametrize("N,d,r", [(1, 1, 1), (2, 3, 1), (5, 4, 2), (8, 4, 2), (8, 2, 0)])
def test_brute_force_tiny(oracle_mod, N, d, r):
    x = _rand(1, 1, N, d, r, seed=50 + N * 10 + d)
    s = 0.7
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"] if r else None,
                            x["w"] if r else None, s)
    bo, bl = _brute(x["q"][0, 0].tolist(), x["k"][0, 0].tolist(), x["v"][0, 0].tolist(),
                    x["u"][0, 0].tolist() if r else None, x["w"][0, 0].tolist() if r else None, s)
    np.testing.assert_allclose(o[0, 0], np.array(bo), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.array(bl), rtol=0, atol=1e-14)


LN2, LN3 = math.log(2.0), math.log(3.0)

# Hand-derived cases.  Each entry: inputs (one head), scale, expected O and LSE.
CLOSED_FORMS = [
    # Scores come from the bias alone: row 0 has bias (0, ln 3) -> P = (1/4, 3/4),
    # O = 1/4 * 1 + 3/4 * 5 = 4, LSE = ln(1 + 3); row 1 has no bias -> P = (1/2, 1/2).
    dict(name="bias_only", scale=1.0, q=[[0.0], [0.0]], k=[[0.0], [0.0]], v=[[1.0], [5.0]],
         u=[[1.0], [0.0]], w=[[0.0], [LN3]], o=[[4.0], [3.0]], lse=[math.log(4), LN2]),
    # Content only, s = 1/2: row scores (0, ln2, 0), (0, 0, 0), (0, 0, ln3) ->
    # P = (1/4, 1/2, 1/4), (1/3, 1/3, 1/3), (1/5, 1/5, 3/5).
    dict(name="content_only", scale=0.5, q=[[2.0, 0.0], [0.0, 0.0], [0.0, 2.0]],
         k=[[0.0, 0.0], [LN2, 0.0], [0.0, LN3]], v=[[1.0, 0.0], [0.0, 1.0], [4.0, 4.0]],
         u=None, w=None, o=[[1.25, 1.5], [5 / 3, 5 / 3], [2.6, 2.6]],
         lse=[math.log(4), LN3, math.log(5)]),
    # Bias U W^T with an asymmetric W (W U^T would put ln3 in row 0 instead):
    # row 0 scores (ln2 + 0, 0 + 0) -> P = (2/3, 1/3), O = 4, LSE = ln3;
    # row 1 scores (0 + ln3, 0 + 0) -> P = (3/4, 1/4), O = 3.75, LSE = ln4.
    dict(name="bias_orientation", scale=1.0, q=[[LN2], [0.0]], k=[[1.0], [0.0]],
         v=[[3.0], [6.0]], u=[[1.0, 0.0], [0.0, 1.0]], w=[[0.0, LN3], [0.0, 0.0]],
         o=[[4.0], [3.75]], lse=[LN3, math.log(4)]),
    # s = 1/2 scales Q K^T but not the bias: row 0 scores (1/2 * 2ln2 + 0, 0 + ln3)
    # = (ln2, ln3) -> P = (2/5, 3/5), O = 0.4 + 3.6 = 4, LSE = ln5.
    dict(name="bias_unscaled", scale=0.5, q=[[1.0], [0.0]], k=[[2 * LN2], [0.0]],
         v=[[1.0], [6.0]], u=[[1.0], [0.0]], w=[[0.0], [LN3]], o=[[4.0], [3.5]],
         lse=[math.log(5), LN2]),
]


@pytest.mark.parametrize("case", CLOSED_FORMS, ids=[c["name"] for c in CLOSED_FORMS])
def test_closed_forms(oracle_mod, case):
    c = case
    q, k, v = (np.array(c[n], dtype=np.float64)[None, None] for n in ("q", "k", "v"))
    u = None if c["u"] is None else np.array(c["u"], dtype=np.float64)[None, None]
    w = None if c["w"] is None else np.array(c["w"], dtype=np.float64)[None, None]
    o, lse = oracle_mod.fwd(q, k, v, u, w, c["scale"])
    np.testing.assert_allclose(o[0, 0], np.array(c["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.array(c["lse"]), rtol=0, atol=1e-14)


def test_row_sampling_matches_full(oracle_mod):
    x = _rand(2, 3, 45, 8, 8, seed=21)
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], 0.4)
    rows = [0, 44, 13, 13, 7]
    os_, ls_ = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], 0.4,
                              bh_range=(2, 5), rows=rows)
    of = o.reshape(6, 45, 8)[2:5][:, rows]
    np.testing.assert_array_equal(os_, of)
    np.testing.assert_array_equal(ls_, lse.reshape(6, 45)[2:5][:, rows])


def test_golden_tiny_regression(oracle_mod):
    """Regression lock on the tiny workload, written by tests/golden/make_golden.py
    (which calls only the oracle).  Guards later edits of the oracle."""
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        g = json.load(f)
    from rank_biased_window_b200.inputs import WORKLOADS, workload_inputs
    wl = WORKLOADS["tiny"]
    x = {k: to_f64(v) for k, v in workload_inputs(wl).items()}
    o, lse = oracle_mod.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], wl.scale)
    np.testing.assert_allclose(lse.reshape(-1), np.array(g["lse"]), rtol=0, atol=1e-13)
    for row, vals in g["o_rows"].items():
        np.testing.assert_allclose(o.reshape(-1, wl.d)[int(row)], np.array(vals), rtol=0,
                                   atol=1e-13)
