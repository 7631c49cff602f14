"""GPU invariants, argument rejection through the binding, and the
failure-detection path (a bounded wait that expires on purpose)."""
import math
import threading

import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs
from tests._parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def _dev(x, dev):
    return {k: v.to(dev) for k, v in x.items()}


@pytest.mark.parametrize("N,d,r", [(64, 32, 8), (700, 64, 32)])
def test_identical_value_rows(rfb_lib, cuda_dev, N, d, r):
    x = _dev(make_inputs(2, 2, N, d, r, seed=3), cuda_dev)
    v = x["v"][:, :, :1, :].expand_as(x["v"]).contiguous()
    o, _ = rfb_lib.attn_fwd(x["q"], x["k"], v, x["u"], x["w"], 1 / math.sqrt(d))
    assert_close("O", o, to_np(v))


@pytest.mark.parametrize("N,d,r", [(64, 32, 8), (500, 64, 32)])
def test_row_constant_bias(rfb_lib, cuda_dev, N, d, r):
    """All W_j equal: O equals the unbiased output, LSE shifts by U_i . w."""
    x = _dev(make_inputs(1, 3, N, d, r, seed=4), cuda_dev)
    w = x["w"][:, :, :1, :].expand_as(x["w"]).contiguous()
    s = 1 / math.sqrt(d)
    o_b, l_b = rfb_lib.attn_fwd(x["q"], x["k"], x["v"], x["u"], w, s)
    o_0, l_0 = rfb_lib.attn_fwd(x["q"], x["k"], x["v"], None, None, s)
    assert_close("O", o_b, to_np(o_0))
    shift = (x["u"].double() * w[:, :, :1, :].double()).sum(-1)
    assert_close("LSE shift", (l_b - l_0).double(), to_np(shift))


def test_key_permutation(rfb_lib, cuda_dev):
    x = _dev(make_inputs(1, 2, 384, 64, 32, seed=6), cuda_dev)
    perm = torch.randperm(384, generator=torch.Generator().manual_seed(0)).to(cuda_dev)
    s = 0.125
    o1, l1 = rfb_lib.attn_fwd(x["q"], x["k"], x["v"], x["u"], x["w"], s)
    o2, l2 = rfb_lib.attn_fwd(x["q"], x["k"][:, :, perm].contiguous(),
                              x["v"][:, :, perm].contiguous(), x["u"],
                              x["w"][:, :, perm].contiguous(), s)
    assert_close("O", o2, to_np(o1))
    assert_close("LSE", l2, to_np(l1))


def test_empty_inputs_are_noops(rfb_lib, cuda_dev):
    q = torch.empty((0, 2, 64, 32), dtype=torch.bfloat16, device=cuda_dev)
    o, lse = rfb_lib.attn_fwd(q, q, q, None, None, 0.5)
    assert o.numel() == 0 and lse.numel() == 0
    z = torch.empty((1, 1, 0, 32), dtype=torch.bfloat16, device=cuda_dev)
    o, lse = rfb_lib.attn_fwd(z, z, z, None, None, 0.5)
    assert o.numel() == 0


def test_argument_rejection(rfb_lib, cuda_dev):
    x = _dev(make_inputs(1, 1, 64, 32, 8, seed=1), cuda_dev)
    lib = rfb_lib.load_library()
    import ctypes
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device=cuda_dev)
    o = torch.empty_like(x["q"])
    lp = ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
    args = [p(x["q"]), p(x["k"]), p(x["v"]), p(x["u"]), p(x["w"]), p(o), lp]
    # unsupported head dimension / rank
    assert lib.rfb_attn_fwd(*args, 1, 1, 64, 48, 8, 0.1, None) == 2
    assert lib.rfb_attn_fwd(*args, 1, 1, 64, 32, 12, 0.1, None) == 2
    # misaligned pointer (2-byte offset into q)
    bad = list(args)
    bad[0] = ctypes.c_void_p(x["q"].data_ptr() + 2)
    assert lib.rfb_attn_fwd(*bad, 1, 1, 64, 32, 8, 0.1, None) == 3
    # null u with r > 0, non-finite scale, negative size
    bad = list(args)
    bad[3] = None
    assert lib.rfb_attn_fwd(*bad, 1, 1, 64, 32, 8, 0.1, None) == 1
    assert lib.rfb_attn_fwd(*args, 1, 1, 64, 32, 8, float("nan"), None) == 1
    assert lib.rfb_attn_fwd(*args, 1, -1, 64, 32, 8, 0.1, None) == 1
    # too-small workspace
    with pytest.raises(RuntimeError, match="workspace"):
        rfb_lib.attn_bwd(x["q"], x["k"], x["v"], x["u"], x["w"], o, lse, x["q"], 0.1,
                         workspace=torch.empty(64, dtype=torch.uint8, device=cuda_dev))
    with pytest.raises(TypeError):
        rfb_lib.attn_fwd(x["q"].float(), x["k"], x["v"], x["u"], x["w"])


def test_wait_timeout_is_reported_and_recoverable(rfb_lib, cuda_dev):
    """A bounded wait on a barrier nothing arrives at expires after ~2 ms, sets
    the device error word (status 6, site 99) and leaves the context usable."""
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    rfb_lib.selftest_wait_timeout(2000)
    err = rfb_lib.last_device_error()
    assert err & 0xFF == 6 and (err >> 8) == 99, err
    assert rfb_lib.last_device_error() == 0  # cleared by the read
    x = _dev(make_inputs(1, 1, 64, 32, 8, seed=2), cuda_dev)
    o, _ = rfb_lib.attn_fwd(x["q"], x["k"], x["v"], x["u"], x["w"], 0.2)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert rfb_lib.last_device_error() == 0


def test_call_from_another_thread(rfb_lib, oracle_mod, cuda_dev):
    """The C ABI works from any host thread (torch runs autograd backward on its
    own device thread)."""
    from rank_biased_window_b200.inputs import to_f64
    x = make_inputs(1, 2, 96, 32, 8, seed=8, with_dout=True)
    out = {}

    def work():
        try:
            torch.cuda.set_device(cuda_dev)
            g = _dev(x, cuda_dev)
            o, lse = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], g["u"], g["w"], 0.25)
            out["grads"] = rfb_lib.attn_bwd(g["q"], g["k"], g["v"], g["u"], g["w"], o, lse,
                                            g["dout"], 0.25)
            out["o"] = o
            torch.cuda.synchronize()
        except Exception as e:  # noqa: BLE001
            out["error"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    if "error" in out:
        raise out["error"]
    f = {k: to_f64(v) for k, v in x.items()}
    ro, _ = oracle_mod.fwd(f["q"], f["k"], f["v"], f["u"], f["w"], 0.25)
    assert_close("O", out["o"], ro)
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], f["u"], f["w"], f["dout"], 0.25)
    for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), out["grads"], ref):
        assert_close(name, got, want)


def test_software_exp2_accuracy(rfb_lib, cuda_dev):
    """The software 2^x used for part of the softmax exponentials: relative
    error against the exact value below 1e-4 on [-125, 10], and about 2^-125
    for inputs below -125 (negligible against any row sum of the softmax)."""
    x = torch.cat([torch.linspace(-125.0, 10.0, 200001), torch.tensor([-0.5, 0.0, 0.5, 1.0, -124.9])])
    y = rfb_lib.binding.selftest_soft_exp2(x.to(cuda_dev)).cpu().double()
    exact = torch.exp2(x.double())
    rel = ((y - exact).abs() / exact).max().item()
    assert rel < 1e-4, rel
    low = rfb_lib.binding.selftest_soft_exp2(torch.tensor([-200.0, -1e30, float("-inf")],
                                                          device=cuda_dev)).cpu().double()
    assert torch.all((low / 2.0 ** -125 - 1).abs() < 1e-4)
