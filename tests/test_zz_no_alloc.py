"""The backward entry point that allocates nothing, rfb_attn_bwd_noalloc.

It exists for callers that may not allocate device memory while they run and
cannot lend the library a workspace (a serving runtime that reserved all device
memory at start-up, a plugin host that owns the allocator).  Its scratch is a
fixed array compiled into the library, shared by every call on a device.

The test calls it through the C ABI twice in a row and compares each result
with the regular workspace-taking backward, within the tolerance the parity
tests use.  The second call checks that what the first call left in the shared
array does not leak into the next result.  This file is named so that pytest
collects it last.
"""
import ctypes

import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs
from tests._parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, g, o, lse, grads, shape, scale):
    B, H, N, d, r = shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    lp = ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
    dq, dk, dv, du, dw = grads
    return lib.rfb_attn_bwd_noalloc(
        p(g["q"]), p(g["k"]), p(g["v"]), p(g["u"] if r else None), p(g["w"] if r else None),
        p(o), lp, p(g["dout"]), p(dq), p(dk), p(dv), p(du), p(dw), B, H, N, d, r, scale,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("shape", [(1, 2, 300, 64, 32), (2, 3, 64, 32, 8), (1, 1, 129, 64, 0)])
def test_noalloc_backward_matches_workspace_backward(rfb_lib, cuda_dev, shape):
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=3100 + N + r, with_dout=True)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    s = d ** -0.5
    u = g["u"] if r else None
    w = g["w"] if r else None
    o, lse = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], u, w, s)
    ref = rfb_lib.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], s)
    lib = rfb_lib.load_library()
    for call in range(2):
        grads = [torch.full_like(g["q"], float("nan")), torch.full_like(g["k"], float("nan")),
                 torch.full_like(g["v"], float("nan")),
                 torch.full_like(g["u"], float("nan")) if r else None,
                 torch.full_like(g["w"], float("nan")) if r else None]
        rc = _call_noalloc(lib, g, o, lse, grads, shape, s)
        assert rc == 0, rfb_lib.strerror(rc)
        torch.cuda.synchronize()
        assert rfb_lib.last_device_error() == 0
        for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), grads, ref):
            if want is None:
                continue
            assert_close(f"call {call + 1} {name}", got, to_np(want))


def test_noalloc_rejects_problems_beyond_its_scratch(rfb_lib, cuda_dev):
    """B=2, H=8, N=16384, d=64, r=32 needs ~100 MB of scratch, more than the
    fixed 32 MiB: rejected on the host (status 4) before anything is enqueued."""
    lib = rfb_lib.load_library()
    need = rfb_lib.bwd_workspace_size(2, 8, 16384, 64, 32)
    assert need > rfb_lib.binding.NOALLOC_SCRATCH_BYTES
    t = torch.zeros(64, dtype=torch.bfloat16, device=cuda_dev)
    lse = torch.zeros(64, dtype=torch.float32, device=cuda_dev)
    p = ctypes.c_void_p(t.data_ptr())
    lp = ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float))
    rc = lib.rfb_attn_bwd_noalloc(p, p, p, p, p, p, lp, p, p, p, p, p, p, 2, 8, 16384, 64, 32,
                                  0.125, None)
    assert rc == 4
