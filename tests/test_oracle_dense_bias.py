"""Pins of the oracle's dense-bias forward (the materialised-bias form used by
the comparator kernel) against the independently written factored oracle."""
import numpy as np
import pytest

import oracle
from rank_biased_window_b200.inputs import make_inputs, to_f64


def test_dense_bias_equals_factored_oracle():
    """Bias = U W^T formed in float64 must give the factored oracle's result
    (two separate implementations: numpy here, C for the factored one)."""
    B, H, N, d, r = 2, 3, 40, 16, 8
    x = make_inputs(B, H, N, d, r, seed=901)
    f = {k: to_f64(v) for k, v in x.items()}
    bias = np.einsum("bhnr,bhmr->bhnm", f["u"], f["w"])
    o1, l1 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], bias, 0.3)
    o2, l2 = oracle.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], 0.3)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-12)


def test_dense_bias_shared_per_head_and_zero_bias():
    B, H, N, d = 3, 2, 24, 8
    x = make_inputs(B, H, N, d, 4, seed=902)
    f = {k: to_f64(v) for k, v in x.items()}
    # one matrix per head == the same matrix repeated for every window
    bh = np.einsum("hnr,hmr->hnm", f["u"][0], f["w"][0])
    o1, l1 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], bh, 0.5)
    o2, l2 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], np.broadcast_to(bh, (B, H, N, N)), 0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # zero bias is plain attention: the factored oracle with r = 0
    o3, l3 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], np.zeros((H, N, N)), 0.5)
    o4, l4 = oracle.fwd(f["q"], f["k"], f["v"], None, None, 0.5)
    np.testing.assert_allclose(o3, o4, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l3, l4, rtol=1e-12, atol=1e-12)


def test_dense_bias_row_constant_shift():
    """A bias constant along each row leaves O unchanged and shifts LSE by it."""
    B, H, N, d = 1, 2, 16, 8
    x = make_inputs(B, H, N, d, 0, seed=903)
    f = {k: to_f64(v) for k, v in x.items()}
    c = np.linspace(-2.0, 3.0, N)
    bias = np.broadcast_to(c[None, :, None], (H, N, N))
    o1, l1 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], bias, 0.4)
    o2, l2 = oracle.fwd_dense_bias(f["q"], f["k"], f["v"], np.zeros((H, N, N)), 0.4)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2 + c[None, None, :], rtol=1e-12, atol=1e-12)


# Mistakes planted in a copy of fwd_dense_bias must fail one of the pins above.
MUTANTS = [
    ("bias_transposed", "S = scale * (q[b, h] @ k[b, h].T) + bm", "S = scale * (q[b, h] @ k[b, h].T) + bm.T"),
    ("bias_scaled", "S = scale * (q[b, h] @ k[b, h].T) + bm", "S = scale * (q[b, h] @ k[b, h].T + bm)"),
    ("bias_of_another_head", "bm = bias[h] if bias.ndim == 3 else bias[b, h]",
     "bm = bias[0] if bias.ndim == 3 else bias[b, 0]"),
    ("lse_without_max", "L[b, h] = (m + np.log(l))[:, 0]", "L[b, h] = np.log(l)[:, 0]"),
]


def _planted(old, new):
    import inspect
    src = inspect.getsource(oracle.fwd_dense_bias)
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<planted>", "exec"), ns)
    return ns["fwd_dense_bias"]


def _pins_hold(fn, monkeypatch):
    monkeypatch.setattr(oracle, "fwd_dense_bias", fn)
    try:
        test_dense_bias_equals_factored_oracle()
        test_dense_bias_shared_per_head_and_zero_bias()
        test_dense_bias_row_constant_shift()
    except AssertionError:
        return False
    return True


def test_pins_hold_for_the_unmodified_copy(monkeypatch):
    assert _pins_hold(_planted("L[b, h] =", "L[b, h] ="), monkeypatch)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, monkeypatch):
    assert not _pins_hold(_planted(old, new), monkeypatch), name
