"""GPU parity of the backward kernels against the fp64 oracle (same bf16 inputs,
the GPU forward's O and LSE feeding the GPU backward, exactly as in training)."""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import WORKLOADS, make_inputs, to_f64, workload_inputs
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _gpu_fwd_bwd(rfb, x, dev, scale, r):
    g = {k: v.to(dev) for k, v in x.items()}
    u = g["u"] if r else None
    w = g["w"] if r else None
    o, lse = rfb.attn_fwd(g["q"], g["k"], g["v"], u, w, scale)
    grads = rfb.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], scale)
    torch.cuda.synchronize()
    assert rfb.last_device_error() == 0
    return o, lse, grads


CASES = [
    (1, 1, 64, 32, 8),
    (1, 2, 49, 32, 8),
    (1, 1, 1, 64, 32),
    (2, 1, 128, 64, 32),
    (1, 2, 129, 32, 16),
    (1, 1, 300, 64, 32),
    (1, 1, 256, 64, 0),
    (1, 1, 384, 32, 64),
    (1, 1, 200, 64, 24),
    (1, 1, 200, 64, 64),   # dQ|dU share the S^T columns (no room for their own)
    (1, 2, 130, 64, 16),
    (3, 1, 64, 32, 0),
    # windows of <= 128 tokens with d = 32, r <= 16 (the window backward)
    (2, 3, 100, 32, 16),
    (5, 1, 33, 32, 8),
    (4, 6, 64, 32, 16),
    (2, 2, 128, 32, 0),
]


@pytest.mark.parametrize("shape", CASES, ids=[f"B{b}H{h}N{n}d{d}r{r}" for b, h, n, d, r in CASES])
def test_backward_matches_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=2000 + N + d + r, with_dout=True)
    s = 1.0 / math.sqrt(d)
    _, _, (dq, dk, dv, du, dw) = _gpu_fwd_bwd(rfb_lib, x, cuda_dev, s, r)
    f = {k: to_f64(v) for k, v in x.items()}
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], f["u"] if r else None, f["w"] if r else None,
                         f["dout"], s)
    for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), (dq, dk, dv, du, dw), ref):
        if want is None:
            assert got is None
            continue
        assert_close(name, got, want)


def test_train_workload_backward_sampled(rfb_lib, oracle_mod, cuda_dev):
    """The training workload (B=2, N=16384, H=8, d=64, r=32) at full size:
    dQ / dU compared on sampled query rows of several heads (the oracle computes
    each row on its own), dK / dV / dW compared on all key rows of one head."""
    wl = WORKLOADS["train"]
    x = workload_inputs(wl)
    _, _, (dq, dk, dv, du, dw) = _gpu_fwd_bwd(rfb_lib, x, cuda_dev, wl.scale, wl.r)
    f = {k: to_f64(v) for k, v in x.items()}
    BH, N, d, r = wl.B * wl.H, wl.N, wl.d, wl.r
    rng = np.random.default_rng(11)
    rows = sorted(set(rng.choice(N, size=10, replace=False).tolist()) | {0, N - 1})
    gq, gu, rq, ru = [], [], [], []
    for h in (0, 5, BH - 1):
        q1, u1, _ = oracle_mod.bwd_query_rows(f["q"], f["k"], f["v"], f["u"], f["w"], f["dout"],
                                              wl.scale, h, rows)
        gq.append(dq.reshape(BH, N, d)[h, rows].double().cpu().numpy())
        gu.append(du.reshape(BH, N, r)[h, rows].double().cpu().numpy())
        rq.append(q1)
        ru.append(u1)
    assert_close("dQ (sampled rows)", np.stack(gq), np.stack(rq))
    assert_close("dU (sampled rows)", np.stack(gu), np.stack(ru))
    h = 3
    _, rk, rv, _, rw = oracle_mod.bwd(f["q"], f["k"], f["v"], f["u"], f["w"], f["dout"],
                                      wl.scale, bh_range=(h, h + 1))
    assert_close("dK (one head)", dk.reshape(BH, N, d)[h], rk[0])
    assert_close("dV (one head)", dv.reshape(BH, N, d)[h], rv[0])
    assert_close("dW (one head)", dw.reshape(BH, N, r)[h], rw[0])
    for t in (dq, dk, dv, du, dw):
        assert torch.isfinite(t.float()).all()


def test_backward_properties_any_size(rfb_lib, cuda_dev):
    """Properties that hold at any size: sum_j dV_j = sum_i dO_i, and
    sum_j dK_j = sum_j dW_j = 0 (each row of dS sums to zero)."""
    B, H, N, d, r = 1, 2, 2048, 64, 32
    x = make_inputs(B, H, N, d, r, seed=77, with_dout=True)
    _, _, (dq, dk, dv, du, dw) = _gpu_fwd_bwd(rfb_lib, x, cuda_dev, 0.125, r)
    sdo = x["dout"].double().sum(dim=2)
    sdv = dv.double().cpu().sum(dim=2)
    assert torch.allclose(sdv, sdo, atol=0.5, rtol=2e-2), (sdv - sdo).abs().max()
    scale_k = dk.double().cpu().abs().sum(dim=2)
    assert (dk.double().cpu().sum(dim=2).abs() <= 0.05 * scale_k + 1e-3).all()
    assert (dw.double().cpu().sum(dim=2).abs() <= 0.05 * dw.double().cpu().abs().sum(dim=2)
            + 1e-3).all()


def test_autograd_function(rfb_lib, oracle_mod, cuda_dev):
    B, H, N, d, r = 1, 2, 96, 32, 8
    x = make_inputs(B, H, N, d, r, seed=31, with_dout=True)
    g = {k: v.to(cuda_dev).requires_grad_(k != "dout") for k, v in x.items()}
    o = rfb_lib.rfb_attention(g["q"], g["k"], g["v"], g["u"], g["w"])
    o.backward(g["dout"])
    f = {k: to_f64(v) for k, v in x.items()}
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], f["u"], f["w"], f["dout"], 1 / math.sqrt(d))
    for name, t, want in zip("qkvuw", (g["q"], g["k"], g["v"], g["u"], g["w"]), ref):
        assert_close("d" + name, t.grad, want)


def test_swinir_shaped_window_backward(rfb_lib, oracle_mod, cuda_dev):
    """64 SwinIR-style 8 x 8 windows, 6 heads, d = 32, r = 8 (the window
    backward, two windows per tile): every gradient against the oracle."""
    B, H, N, d, r = 64, 6, 64, 32, 8
    x = make_inputs(B, H, N, d, r, seed=2600, with_dout=True)
    s = 1.0 / math.sqrt(d)
    _, _, grads = _gpu_fwd_bwd(rfb_lib, x, cuda_dev, s, r)
    f = {k: to_f64(v) for k, v in x.items()}
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], f["u"], f["w"], f["dout"], s)
    for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), grads, ref):
        assert_close(name, got, want)
