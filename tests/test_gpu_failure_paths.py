"""Failure paths of the production kernels, without any GPU fault.

1. Abort path: the test hook rfb_debug_set_wait_limit names one wait site of
   the window forward, the long forward or the backward that gives up at once,
   as if its bounded wait had expired.  The kernel must record
   RFB_ERR_DEVICE_TIMEOUT with that site in the error word, let its in-flight
   copies and MMAs land, free TMEM and return; the next normal call on the same
   context must match the fp64 oracle.
2. A very short main-loop wait limit (1 us) on a larger problem: each call
   either completes (and then matches the oracle) or reports a timeout; the
   context stays usable either way.
3. Ragged sizes write nothing outside their tensors: every output (and the
   backward's workspace) sits between two canary regions that must be
   unchanged afterwards.
"""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs, to_f64
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def _dev(x, dev):
    return {k: v.to(dev) for k, v in x.items()}


def _fwd_bwd(rfb, g, scale, r, backward=True):
    u, w = (g["u"], g["w"]) if r else (None, None)
    o, lse = rfb.attn_fwd(g["q"], g["k"], g["v"], u, w, scale)
    grads = rfb.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], scale) \
        if backward else None
    return o, lse, grads


def _check_against_oracle(oracle, x, o, lse, grads, scale, r):
    f = {k: to_f64(v) for k, v in x.items()}
    u, w = (f["u"], f["w"]) if r else (None, None)
    ro, rl = oracle.fwd(f["q"], f["k"], f["v"], u, w, scale)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)
    if grads is not None:
        ref = oracle.bwd(f["q"], f["k"], f["v"], u, w, f["dout"], scale)
        for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), grads, ref):
            if want is not None:
                assert_close(name, got, want)


# (shape, wait sites that every CTA of that kernel reaches)
#   window forward (N <= 128): 2 score MMA waits for its inputs, 3 PV MMA waits
#     for P, 5 softmax waits for S, 6 epilogue waits for O
#   long forward: 12 MMA warps wait for Q, 13 for K / V, 14 for their previous
#     PV, 15 for P, 16 softmax waits for S, 19 for the unit's last PV, 21 for
#     the other key half's row statistics
#   backward: 32 MMA warp waits for K / V, 33 for Q / dO, 35 for dS, 38 softmax
#     waits for S / dP, 39 dQ | dU reduction waits for its MMAs,
#     43 softmax waits for the dS buffer's reductions (three or more query
#     tiles), 44 for the last gradient MMAs
#   window backward (d = 32, N <= 128): 52 MMA warp waits for its stage, 54 for
#     dS, 56 compute warps wait for their stage, 57 for S / dP, 59 for the
#     gradient MMAs
ABORT_CASES = [
    ((1, 2, 64, 32, 8), "fwd", (2, 3, 5, 6)),
    ((1, 2, 300, 64, 32), "fwd", (12, 13, 14, 15, 16, 19, 21)),
    ((1, 1, 777, 32, 16), "fwd", (13, 16)),
    ((1, 2, 300, 64, 32), "bwd", (32, 33, 35, 38, 39, 43, 44)),
    ((2, 1, 64, 32, 8), "bwd", (52, 54, 56, 57, 59)),
    ((1, 2, 100, 32, 0), "bwd", (52, 57, 59)),
]


@pytest.mark.parametrize("case", ABORT_CASES,
                         ids=[f"{k}-N{s[2]}d{s[3]}r{s[4]}" for s, k, _ in ABORT_CASES])
def test_kernel_abort_path_reports_and_recovers(rfb_lib, oracle_mod, cuda_dev, case):
    shape, kernel, sites = case
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=5100 + N + r, with_dout=True)
    g = _dev(x, cuda_dev)
    s = 1.0 / math.sqrt(d)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    try:
        for site in sites:
            if kernel == "bwd":
                o, lse, _ = _fwd_bwd(rfb_lib, g, s, r, backward=False)
                torch.cuda.synchronize()
                rfb_lib.debug_set_wait_limit(0, site)
                u, w = (g["u"], g["w"]) if r else (None, None)
                rfb_lib.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], s)
            else:
                rfb_lib.debug_set_wait_limit(0, site)
                _fwd_bwd(rfb_lib, g, s, r, backward=False)
            rfb_lib.debug_set_wait_limit(0, -1)
            err = rfb_lib.last_device_error()   # synchronises, then clears the word
            assert err & 0xFF == TIMEOUT and err >> 8 == site, (site, hex(err))
    finally:
        rfb_lib.debug_set_wait_limit(0, -1)
    # the same context still computes correct results
    o, lse, grads = _fwd_bwd(rfb_lib, g, s, r, backward=(kernel == "bwd"))
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    _check_against_oracle(oracle_mod, x, o, lse, grads, s, r)


def test_short_wait_limit_completes_or_reports(rfb_lib, oracle_mod, cuda_dev):
    """With every main-loop wait limited to 1 us, a forward + backward on 2 x
    2048 tokens either finishes (results checked) or records a timeout; then,
    back at the default limit, the same call matches the oracle."""
    B, H, N, d, r = 1, 2, 2048, 64, 32
    x = make_inputs(B, H, N, d, r, seed=5200, with_dout=True)
    g = _dev(x, cuda_dev)
    s = 0.125
    outcomes = []
    try:
        rfb_lib.debug_set_wait_limit(1, -1)
        for _ in range(3):
            o, lse, grads = _fwd_bwd(rfb_lib, g, s, r)
            err = rfb_lib.last_device_error()
            assert err == 0 or err & 0xFF == TIMEOUT, hex(err)
            outcomes.append(err)
    finally:
        rfb_lib.debug_set_wait_limit(0, -1)
    if outcomes[-1] == 0:
        _check_against_oracle(oracle_mod, x, o, lse, grads, s, r)
    o, lse, grads = _fwd_bwd(rfb_lib, g, s, r)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    _check_against_oracle(oracle_mod, x, o, lse, grads, s, r)
    print("error words under a 1 us limit:", [hex(e) for e in outcomes])


PAD = 4096  # elements of canary on each side (a multiple of 16 bytes for every dtype)


def _padded(shape, dtype, dev, fill_bits):
    """A contiguous tensor of `shape` in the middle of a larger buffer whose
    PAD elements on each side hold the bit pattern fill_bits."""
    n = int(np.prod(shape))
    itype = torch.int16 if dtype == torch.bfloat16 else torch.int32
    buf = torch.full((n + 2 * PAD,), fill_bits, dtype=itype, device=dev).view(dtype)
    return buf, buf[PAD:PAD + n].view(shape)


def _canaries_intact(buf, fill_bits):
    itype = torch.int16 if buf.dtype == torch.bfloat16 else torch.int32
    raw = buf.view(itype)
    return bool((raw[:PAD] == fill_bits).all() and (raw[-PAD:] == fill_bits).all())


@pytest.mark.parametrize("shape", [(1, 2, 129, 64, 32), (1, 1, 300, 32, 16), (2, 1, 777, 64, 8),
                                   (3, 1, 49, 32, 8), (1, 1, 100, 64, 0)],
                         ids=lambda s: "B{}H{}N{}d{}r{}".format(*s))
def test_ragged_outputs_write_nothing_outside(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=5300 + N, with_dout=True)
    g = _dev(x, cuda_dev)
    s = 1.0 / math.sqrt(d)
    bf_bits, f_bits = 0x7FC1, 0x7FC00001          # NaN patterns no kernel writes
    o_buf, o = _padded((B, H, N, d), torch.bfloat16, cuda_dev, bf_bits)
    l_buf, lse = _padded((B, H, N), torch.float32, cuda_dev, f_bits)
    u, w = (g["u"], g["w"]) if r else (None, None)
    rfb_lib.attn_fwd(g["q"], g["k"], g["v"], u, w, s, out=o, lse=lse)
    grad_bufs, grads = [], []
    for shp in [(B, H, N, d)] * 3 + ([(B, H, N, r)] * 2 if r else []):
        b_, t_ = _padded(shp, torch.bfloat16, cuda_dev, bf_bits)
        grad_bufs.append(b_)
        grads.append(t_)
    if not r:
        grads += [None, None]
    ws_bytes = rfb_lib.bwd_workspace_size(B, H, N, d, r)
    ws_buf, ws = _padded((ws_bytes // 4,), torch.float32, cuda_dev, f_bits)
    out = rfb_lib.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], s,
                           workspace=ws.view(torch.uint8), grads=tuple(grads))
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    assert _canaries_intact(o_buf, bf_bits) and _canaries_intact(l_buf, f_bits)
    for i, b_ in enumerate(grad_bufs):
        assert _canaries_intact(b_, bf_bits), f"gradient {i} wrote outside its tensor"
    assert _canaries_intact(ws_buf, f_bits), "the backward wrote outside its workspace"
    _check_against_oracle(oracle_mod, x, o, lse, out, s, r)
