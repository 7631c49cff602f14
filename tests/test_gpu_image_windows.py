"""GPU parity of shifted-window attention gathered straight from feature maps
against the oracle's step-by-step version (roll, partition, masked window
attention, reverse)."""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs, to_f64
from tests._parity import MAX_ABS, assert_close

pytestmark = pytest.mark.gpu


def _maps(B, Hs, Ws, nh, d, r, seed):
    x = make_inputs(1, B * Hs * Ws, nh, d, r, seed=seed)
    t = {k: v[0] for k, v in x.items()}
    q, k, v = (t[n].reshape(B, Hs, Ws, nh, d).contiguous() for n in ("q", "k", "v"))
    u = t["u"][:64].transpose(0, 1).contiguous() if r else None     # [heads, 64, r]
    w = t["w"][:64].transpose(0, 1).contiguous() if r else None
    return q, k, v, u, w


CASES = [
    (2, 16, 24, 3, 32, 16, 0),
    (2, 16, 24, 3, 32, 16, 4),   # shifted: masks in the last window row and column
    (1, 8, 8, 2, 64, 8, 4),      # one window: four regions
    (1, 24, 16, 6, 32, 8, 4),    # SwinIR-like heads
    (2, 16, 16, 1, 64, 0, 4),    # no bias
    (1, 8, 16, 5, 32, 32, 4),    # odd window-head count: last tile half empty
]


@pytest.mark.parametrize("shape", CASES, ids=[f"B{b}H{hs}W{ws}h{nh}d{d}r{r}s{sh}"
                                              for b, hs, ws, nh, d, r, sh in CASES])
def test_image_windows_match_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, Hs, Ws, nh, d, r, shift = shape
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=8100 + Hs + Ws + d + r + shift)
    s = 1.0 / math.sqrt(d)
    dev = lambda t: None if t is None else t.to(cuda_dev)
    o, lse = rfb_lib.attn_fwd_image_windows(dev(q), dev(k), dev(v), dev(u), dev(w), s,
                                            shift=shift)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    f = lambda t: None if t is None else to_f64(t)
    ro, rl = oracle_mod.fwd_image_windows(f(q), f(k), f(v), f(u), f(w), s, 8, shift)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)


def test_unshifted_maps_equal_partitioned_windows(rfb_lib, cuda_dev):
    """Without a shift the map path equals the window path on windows
    partitioned by reshapes (same kernels' arithmetic; token order inside a
    window differs, which attention does not see)."""
    B, Hs, Ws, nh, d, r = 2, 16, 24, 3, 32, 16
    q, k, v, u, w = (t.to(cuda_dev) for t in _maps(B, Hs, Ws, nh, d, r, seed=8200))
    o, lse = rfb_lib.attn_fwd_image_windows(q, k, v, u, w)

    def part(x):
        c = x.shape[-1]
        x = x.reshape(B, Hs // 8, 8, Ws // 8, 8, nh, c).permute(0, 1, 3, 5, 2, 4, 6)
        return x.reshape(-1, nh, 64, c).contiguous()

    o2, l2 = rfb_lib.attn_fwd_shared_bias(part(q), part(k), part(v), u, w)
    assert (part(o).float() - o2.float()).abs().max().item() < 1e-2
    assert (part(lse[..., None])[..., 0] - l2).abs().max().item() < 1e-3


def test_image_windows_reject_unsupported(rfb_lib, cuda_dev):
    q, k, v, u, w = (t.to(cuda_dev) for t in _maps(1, 12, 16, 2, 32, 8, seed=1))
    with pytest.raises(RuntimeError, match="unsupported"):
        rfb_lib.attn_fwd_image_windows(q, k, v, u, w)           # 12 rows: not whole windows
    q, k, v, u, w = (t.to(cuda_dev) for t in _maps(1, 16, 16, 2, 32, 8, seed=2))
    with pytest.raises(RuntimeError, match="unsupported"):
        rfb_lib.attn_fwd_image_windows(q, k, v, u, w, shift=2)


BWD_CASES = [
    (2, 16, 24, 3, 32, 16, 0),
    (2, 16, 24, 3, 32, 16, 4),   # masks in the last window row and column
    (1, 8, 8, 2, 64, 8, 4),      # one window: four regions
    (1, 24, 16, 6, 32, 8, 4),    # SwinIR-like heads
    (2, 16, 16, 1, 64, 0, 4),    # no bias
    (1, 16, 16, 2, 64, 32, 4),
    (2, 32, 32, 6, 32, 8, 4),    # 32 windows x 6 heads, SwinIR-sized windows
    (1, 16, 24, 2, 32, 0, 4),    # d = 32 without bias
]


@pytest.mark.parametrize("shape", BWD_CASES, ids=[f"B{b}H{hs}W{ws}h{nh}d{d}r{r}s{sh}"
                                                  for b, hs, ws, nh, d, r, sh in BWD_CASES])
def test_image_windows_backward_match_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, Hs, Ws, nh, d, r, shift = shape
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=8300 + Hs + Ws + d + r + shift)
    g = torch.Generator().manual_seed(8400 + Hs + d + shift)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    s = 1.0 / math.sqrt(d)
    dev = lambda t: None if t is None else t.to(cuda_dev)
    o, lse = rfb_lib.attn_fwd_image_windows(dev(q), dev(k), dev(v), dev(u), dev(w), s,
                                            shift=shift)
    got = rfb_lib.attn_bwd_image_windows(dev(q), dev(k), dev(v), dev(u), dev(w), o, lse, dev(do),
                                         s, shift=shift)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    f = lambda t: None if t is None else to_f64(t)
    want = oracle_mod.bwd_image_windows(f(q), f(k), f(v), f(u), f(w), f(do), s, 8, shift)
    for name, a, b in zip(("dQ", "dK", "dV", "dU", "dW"), got, want):
        if b is None:
            assert a is None
            continue
        # dU, dW are sums over all windows of a map (magnitudes up to ~8 here):
        # the bf16 operands of the tensor-core products (dS, U', W) and the bf16
        # output each carry a relative error of 2^-9, so the absolute bound, set
        # for outputs of order 1, is scaled to one bf16 step at the largest
        # magnitude (2^-7 max|x|); the rel-L2 bound is unchanged.
        ma = MAX_ABS if name in ("dQ", "dK", "dV") else max(MAX_ABS, 2.0 ** -7 * np.abs(b).max())
        assert_close(name, a, b, max_abs=ma)


def test_image_windows_autograd(rfb_lib, oracle_mod, cuda_dev):
    """Gradients through torch autograd (both passes run the CUDA kernels)."""
    B, Hs, Ws, nh, d, r, shift = 1, 16, 24, 2, 32, 16, 4
    q, k, v, u, w = _maps(B, Hs, Ws, nh, d, r, seed=8500)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(8501)).to(torch.bfloat16)
    leaves = [t.to(cuda_dev).requires_grad_() for t in (q, k, v, u, w)]
    o = rfb_lib.rfb_attention_image_windows(*leaves, 0.2, shift)
    o.backward(do.to(cuda_dev))
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    want = oracle_mod.bwd_image_windows(*(to_f64(t) for t in (q, k, v, u, w, do)), 0.2, 8, shift)
    for name, t, b in zip(("dQ", "dK", "dV", "dU", "dW"), leaves, want):
        ma = MAX_ABS if name in ("dQ", "dK", "dV") else max(MAX_ABS, 2.0 ** -7 * np.abs(b).max())
        assert_close(name, t.grad, b, max_abs=ma)
