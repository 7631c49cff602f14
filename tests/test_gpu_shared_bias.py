"""Shared bias factors (one U, W pair per head, used by every window; the form
the implicit-neural-representation bias of "Rank-Factorized Implicit Neural
Bias" (Abstract) takes): GPU parity against the fp64 oracle applied to the
factors broadcast over the windows, which is this variant's definition
(dU[h] = sum_b dU[b, h], dW[h] = sum_b dW[b, h])."""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs, to_f64
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _shared_inputs(B, H, N, d, r, seed):
    """Per-window inputs from the seeded generator; the shared factors are the
    first window's, so every distribution matches the per-window workloads."""
    x = make_inputs(B, H, N, d, r, seed=seed, with_dout=True)
    if r:
        x["u"] = x["u"][0].contiguous()
        x["w"] = x["w"][0].contiguous()
    return x


def _expand(t, B):
    """[H, N, r] -> [B, H, N, r] (torch tensor or numpy array)."""
    if isinstance(t, np.ndarray):
        return np.broadcast_to(t[None], (B,) + t.shape).copy()
    return t.unsqueeze(0).expand(B, *t.shape).contiguous()


CASES = [
    (2, 3, 64, 32, 16),   # two windows per tile whose bias heads wrap (2, 0); resident
    (1, 1, 64, 32, 8),    # one window: as many bias heads as window-heads
    (2, 9, 64, 32, 16),   # too many heads to keep resident: one copy per window, wrapping
    (2, 3, 100, 64, 64),  # one window per tile, copied per window
    (3, 1, 49, 64, 8),    # ragged window
    (2, 2, 200, 64, 32),  # long regime
    (2, 3, 130, 32, 16),
    (4, 1, 128, 64, 64),
    (1, 2, 64, 32, 0),    # no bias: same as the per-window path
    (4, 6, 64, 32, 8),    # window backward, two windows per tile, heads wrapping
    (3, 2, 100, 32, 16),  # window backward, one window per tile
]


@pytest.mark.parametrize("shape", CASES, ids=[f"B{b}H{h}N{n}d{d}r{r}" for b, h, n, d, r in CASES])
def test_shared_bias_matches_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, r = shape
    x = _shared_inputs(B, H, N, d, r, seed=5000 + N + d + r)
    s = 1.0 / math.sqrt(d)
    g = {k: (v.to(cuda_dev) if v is not None else None) for k, v in x.items()}
    u = g["u"] if r else None
    w = g["w"] if r else None
    o, lse = rfb_lib.attn_fwd_shared_bias(g["q"], g["k"], g["v"], u, w, s)
    dq, dk, dv, du, dw = rfb_lib.attn_bwd_shared_bias(g["q"], g["k"], g["v"], u, w, o, lse,
                                                      g["dout"], s)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    f = {k: to_f64(v) for k, v in x.items()}
    ue = _expand(f["u"], B) if r else None
    we = _expand(f["w"], B) if r else None
    ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], ue, we, s)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)
    rq, rk, rv, ru, rw = oracle_mod.bwd(f["q"], f["k"], f["v"], ue, we, f["dout"], s)
    assert_close("dQ", dq, rq)
    assert_close("dK", dk, rk)
    assert_close("dV", dv, rv)
    if r:
        assert du.shape == (H, N, r) and dw.shape == (H, N, r)
        assert_close("dU (sum over windows)", du, ru.sum(axis=0))
        assert_close("dW (sum over windows)", dw, rw.sum(axis=0))
    else:
        assert du is None and dw is None


def test_shared_equals_expanded_per_window(rfb_lib, cuda_dev):
    """The shared entry points compute exactly what the per-window ones do on
    the broadcast factors: O, LSE, dQ, dK, dV bit for bit; dU, dW are the
    window sums (fp32 then rounded, so compared within bf16 rounding)."""
    B, H, N, d, r = 3, 2, 64, 32, 16
    x = _shared_inputs(B, H, N, d, r, seed=61)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    ue, we = _expand(g["u"], B), _expand(g["w"], B)
    o1, l1 = rfb_lib.attn_fwd_shared_bias(g["q"], g["k"], g["v"], g["u"], g["w"])
    o2, l2 = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], ue, we)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    a = rfb_lib.attn_bwd_shared_bias(g["q"], g["k"], g["v"], g["u"], g["w"], o1, l1, g["dout"])
    b = rfb_lib.attn_bwd(g["q"], g["k"], g["v"], ue, we, o2, l2, g["dout"])
    for t1, t2 in zip(a[:3], b[:3]):
        assert torch.equal(t1, t2)
    for t1, t2 in zip(a[3:], b[3:]):
        ref = t2.float().sum(dim=0)
        assert torch.allclose(t1.float(), ref, rtol=2e-2, atol=2e-2 * ref.abs().max().item())
    assert rfb_lib.last_device_error() == 0


def test_shared_bias_autograd(rfb_lib, oracle_mod, cuda_dev):
    B, H, N, d, r = 2, 2, 96, 32, 8
    x = _shared_inputs(B, H, N, d, r, seed=73)
    g = {k: v.to(cuda_dev).requires_grad_(k != "dout") for k, v in x.items()}
    o = rfb_lib.rfb_attention_shared_bias(g["q"], g["k"], g["v"], g["u"], g["w"])
    o.backward(g["dout"])
    f = {k: to_f64(v) for k, v in x.items()}
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], _expand(f["u"], B), _expand(f["w"], B),
                         f["dout"], 1 / math.sqrt(d))
    for name, t, want in zip("qkv", (g["q"], g["k"], g["v"]), ref[:3]):
        assert_close("d" + name, t.grad, want)
    assert_close("du", g["u"].grad, ref[3].sum(axis=0))
    assert_close("dw", g["w"].grad, ref[4].sum(axis=0))


def test_shared_bias_rejects_wrong_factor_shape(rfb_lib, cuda_dev):
    x = make_inputs(2, 2, 64, 32, 8, seed=3, with_dout=False)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    with pytest.raises(ValueError):
        rfb_lib.attn_fwd_shared_bias(g["q"], g["k"], g["v"], g["u"], g["w"])  # [B, H, N, r]
