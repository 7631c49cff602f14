"""A sweep of shapes chosen for the kernels' scheduling paths rather than for
the workloads: many units per persistent CTA in both regimes, units with many
more key tiles than K / V stages (the next unit's Q / U' prepared while the
current unit runs), one unit per CTA, ragged token counts and every padding of
r.  Forward and backward are compared with the fp64 oracle on sampled heads
(all rows for dK / dV / dW, which the oracle computes per head) and sampled
query rows (O, LSE, dQ, dU)."""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs, to_f64
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

# (B, H, N, d, r)
SHAPES = [
    (1, 160, 1700, 32, 8),    # long regime, 14 key tiles per unit, ~8 units per CTA
    (2, 40, 2100, 64, 24),    # d = 64, 17 key tiles, r padded to 32
    (1, 300, 200, 32, 16),    # 2 key tiles per unit, 300 units
    (3, 100, 129, 64, 0),     # one query pair per head, a one-token key tail
    (1, 200, 777, 32, 64),    # d = 32 with r_pad = 64
    (2, 80, 64, 32, 8),       # window regime, 160 window-heads
    (5, 100, 49, 32, 16),     # window regime, ragged 7x7 windows
    (1, 3, 4096, 64, 32),     # one unit per CTA, 32 key tiles
    (1, 2, 3000, 32, 40),     # d = 32, r_pad = 64, 24 key tiles, ragged
    (4, 37, 128, 64, 56),     # N = 128 at d = 64, r_pad = 64
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"B{b}H{h}N{n}d{d}r{r}" for b, h, n, d, r in SHAPES])
def test_shape_sweep_forward_backward(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, r = shape
    BH = B * H
    x = make_inputs(B, H, N, d, r, seed=9000 + N + 3 * H + r, with_dout=True)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    s = 1.0 / math.sqrt(d)
    u, w = (g["u"], g["w"]) if r else (None, None)
    o, lse = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], u, w, s)
    dq, dk, dv, du, dw = rfb_lib.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], s)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    f = {k: to_f64(v) for k, v in x.items()}
    fu, fw = (f["u"], f["w"]) if r else (None, None)
    rng = np.random.default_rng(N + BH)
    heads = sorted(set(rng.choice(BH, size=min(2, BH), replace=False).tolist()) | {BH - 1})
    rows = sorted(set(rng.choice(N, size=min(12, N), replace=False).tolist()) | {0, N - 1})
    og, lg = o.reshape(BH, N, d), lse.reshape(BH, N)
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for h in heads:
        ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], fu, fw, s, bh_range=(h, h + 1), rows=rows)
        got_o.append(og[h, rows].double().cpu().numpy())
        got_l.append(lg[h, rows].double().cpu().numpy())
        ref_o.append(ro[0])
        ref_l.append(rl[0])
    assert_close("O (sampled)", np.stack(got_o), np.stack(ref_o))
    assert_close("LSE (sampled)", np.stack(got_l), np.stack(ref_l))
    # backward: whole heads for the key-side gradients, sampled rows for the
    # query-side ones
    h = heads[-1]
    rq, rk, rv, ru, rw = oracle_mod.bwd(f["q"], f["k"], f["v"], fu, fw, f["dout"], s,
                                        bh_range=(h, h + 1))
    assert_close("dK (one head)", dk.reshape(BH, N, d)[h], rk[0])
    assert_close("dV (one head)", dv.reshape(BH, N, d)[h], rv[0])
    assert_close("dQ (one head)", dq.reshape(BH, N, d)[h], rq[0])
    if r:
        assert_close("dU (one head)", du.reshape(BH, N, r)[h], ru[0])
        assert_close("dW (one head)", dw.reshape(BH, N, r)[h], rw[0])
    for t in (o, lse, dq, dk, dv) + ((du, dw) if r else ()):
        assert torch.isfinite(t.float()).all()
