"""GPU parity of the forward kernels against the fp64 oracle (same bf16 inputs).

Small and ragged cases are compared element by element; the full-size
workloads run in the launch configuration the bench times and are compared on
sampled rows that the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import WORKLOADS, make_inputs, to_f64, workload_inputs
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _run_gpu(rfb, x, dev, scale, r):
    g = {k: v.to(dev) for k, v in x.items()}
    o, lse = rfb.attn_fwd(g["q"], g["k"], g["v"], g["u"] if r else None, g["w"] if r else None,
                          scale)
    torch.cuda.synchronize()
    assert rfb.last_device_error() == 0
    return o, lse


CASES = [
    # (B, H, N, d, r)   window regime (N <= 128): packing, phantom window, ragged N
    (1, 1, 64, 32, 8),     # the tiny workload's shape
    (1, 3, 64, 32, 8),     # odd number of windows: last tile half empty
    (2, 3, 49, 32, 8),     # 7x7 windows (ragged inside the 64-row slot)
    (1, 2, 1, 32, 8),      # one token
    (1, 2, 17, 64, 32),
    (1, 2, 100, 32, 16),   # one window per 128-row tile, ragged
    (1, 1, 128, 64, 64),
    (2, 2, 64, 64, 0),     # no bias
    (1, 2, 64, 32, 24),    # r padded to 32
    (1, 1, 64, 32, 40),    # r padded to 64
    (4, 75, 64, 32, 8),    # 300 windows -> 150 tiles: persistent CTAs loop
    # long regime (N > 128): online softmax over key tiles, ragged tails
    (1, 1, 129, 32, 8),
    (1, 2, 256, 64, 32),
    (2, 1, 300, 32, 16),
    (1, 1, 1000, 64, 0),
    (1, 1, 1024, 32, 16),
    (1, 1, 777, 64, 64),
    # d = 32 with several units (head, query-tile pair) per CTA: the next
    # unit's first scores are issued before the current unit ends
    (8, 50, 300, 32, 16),  # 3 key tiles, ragged
    (4, 100, 200, 32, 8),  # 2 key tiles: the next unit prepared at the last tile
    (2, 100, 257, 32, 0),  # a last query pair of one row
    (1, 40, 1664, 32, 8),  # 13 key tiles per unit (more than twice the K / V stages)
]


@pytest.mark.parametrize("shape", CASES, ids=[f"B{b}H{h}N{n}d{d}r{r}" for b, h, n, d, r in CASES])
def test_forward_matches_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=1000 + N + 7 * d + r)
    s = 1.0 / math.sqrt(d)
    o, lse = _run_gpu(rfb_lib, x, cuda_dev, s, r)
    f = {k: to_f64(v) for k, v in x.items()}
    ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"] if r else None,
                            f["w"] if r else None, s)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)


def test_forward_scale_and_large_scores(rfb_lib, oracle_mod, cuda_dev):
    """A large scale spreads the scores (exercises the running-max rescale)."""
    B, H, N, d, r = 1, 2, 640, 64, 32
    x = make_inputs(B, H, N, d, r, seed=4242)
    s = 0.6
    o, lse = _run_gpu(rfb_lib, x, cuda_dev, s, r)
    f = {k: to_f64(v) for k, v in x.items()}
    ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], s)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl, max_abs=2e-2)


SAMPLED = {
    # workload: (number of heads sampled, rows per head)
    "swinir": (48, 64),
    "large": (6, 48),
    "global": (3, 24),
    "train": (2, 12),
}


@pytest.mark.parametrize("name", ["tiny", "swinir", "large", "global", "train"])
def test_workload_forward(rfb_lib, oracle_mod, cuda_dev, name):
    wl = WORKLOADS[name]
    x = workload_inputs(wl, with_dout=False)
    o, lse = _run_gpu(rfb_lib, x, cuda_dev, wl.scale, wl.r)
    f = {k: to_f64(v) for k, v in x.items()}
    BH, N, d = wl.B * wl.H, wl.N, wl.d
    if name == "tiny":
        ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], wl.scale)
        assert_close("O", o, ro)
        assert_close("LSE", lse, rl)
        return
    nh, nr = SAMPLED[name]
    rng = np.random.default_rng(7)
    heads = sorted(set(rng.choice(BH, size=nh, replace=False).tolist()) | {0, BH - 1})
    rows = sorted(set(rng.choice(N, size=nr, replace=False).tolist()) | {0, N - 1})
    og = o.reshape(BH, N, d)
    lg = lse.reshape(BH, N)
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for h in heads:
        ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], wl.scale,
                                bh_range=(h, h + 1), rows=rows)
        got_o.append(og[h, rows].double().cpu().numpy())
        got_l.append(lg[h, rows].double().cpu().numpy())
        ref_o.append(ro[0])
        ref_l.append(rl[0])
    assert_close(f"{name} O (sampled)", np.stack(got_o), np.stack(ref_o))
    assert_close(f"{name} LSE (sampled)", np.stack(got_l), np.stack(ref_l))
    # every output finite (cheap whole-tensor property)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_repeat_calls_identical(rfb_lib, cuda_dev):
    """The forward is deterministic: two calls give bitwise-identical results."""
    x = make_inputs(2, 3, 300, 64, 32, seed=5)
    o1, l1 = _run_gpu(rfb_lib, x, cuda_dev, 0.125, 32)
    o2, l2 = _run_gpu(rfb_lib, x, cuda_dev, 0.125, 32)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [32, 64])
def test_forward_growing_row_max(rfb_lib, oracle_mod, cuda_dev, d):
    """A bias that ramps along the keys, rising for some query rows and falling
    for others, so that the running max grows past the lazy-rescale threshold
    on every key tile for half the rows of each warp (the tile is exponentiated
    again with the new max and O rescaled) and never for the rest."""
    B, H, N, r = 1, 2, 700, 16
    x = make_inputs(B, H, N, d, r, seed=77 + d)
    n = torch.arange(N, dtype=torch.float32)
    u = torch.zeros(B, H, N, r)
    w = torch.zeros(B, H, N, r)
    u[..., 0] = torch.where(n % 2 == 0, 1.0, -1.0) * (0.5 + (n % 7) / 8.0)
    w[..., 0] = 0.06 * n
    x["u"], x["w"] = u.to(torch.bfloat16), w.to(torch.bfloat16)
    # A power-of-two scale keeps U / s exact in bf16 at these bias magnitudes.
    s = 0.125
    o, lse = _run_gpu(rfb_lib, x, cuda_dev, s, r)
    f = {k: to_f64(v) for k, v in x.items()}
    ro, rl = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], s)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)
