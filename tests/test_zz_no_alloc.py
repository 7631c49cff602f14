"""The backward entry point that allocates nothing, rfb_attn_bwd_noalloc.

It exists for callers that may not allocate device memory while they run and
cannot lend the library a workspace (a serving runtime that reserved all device
memory at start-up, a plugin host that owns the allocator).  Its scratch is a
fixed array compiled into the library, shared by every call on a device.

The tests call it through the C ABI several times in a row and compare each
result with the regular workspace-taking backward on the same inputs, within
the tolerance the parity tests use.  Consecutive calls use different shapes,
seeds and ranks (one of them nearly fills the array), so what one call left
in the shared array would show up in the next result if any part of the
scratch were not rewritten or cleared.  The Python wrapper, the set-up call and
the host-side rejection of problems beyond the array are checked too.  This
file is named so that pytest collects it last.
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


def _problem(rfb, dev, shape, seed):
    """Inputs, forward outputs and the workspace backward's gradients."""
    B, H, N, d, r = shape
    x = make_inputs(B, H, N, d, r, seed=seed, with_dout=True)
    g = {k: v.to(dev) for k, v in x.items()}
    s = d ** -0.5
    u, w = (g["u"], g["w"]) if r else (None, None)
    o, lse = rfb.attn_fwd(g["q"], g["k"], g["v"], u, w, s)
    ref = rfb.attn_bwd(g["q"], g["k"], g["v"], u, w, o, lse, g["dout"], s)
    return g, o, lse, s, ref


def _nan_grads(g, r):
    return [torch.full_like(g["q"], float("nan")), torch.full_like(g["k"], float("nan")),
            torch.full_like(g["v"], float("nan")),
            torch.full_like(g["u"], float("nan")) if r else None,
            torch.full_like(g["w"], float("nan")) if r else None]


def _near_limit_shape(rfb):
    """(1, 4, N, 64, 32) with N the largest multiple of 128 whose scratch fits
    the fixed array (about 97 % of it)."""
    limit = rfb.binding.NOALLOC_SCRATCH_BYTES
    n = 128
    while rfb.bwd_workspace_size(1, 4, n + 128, 64, 32) <= limit:
        n += 128
    return (1, 4, n, 64, 32)


def test_noalloc_setup_call(rfb_lib, cuda_dev):
    """An empty call (B = 0) only loads the kernels and caches the array's
    address; it launches nothing and returns success."""
    lib = rfb_lib.load_library()
    rc = lib.rfb_attn_bwd_noalloc(*([None] * 13), 0, 4, 64, 64, 32, 0.125, None)
    assert rc == 0, rfb_lib.strerror(rc)
    rfb_lib.attn_bwd_noalloc_setup(cuda_dev)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0


def test_noalloc_backward_matches_workspace_backward(rfb_lib, cuda_dev):
    """Calls in a row through the C ABI: a problem that nearly fills the array,
    then smaller ragged ones with other seeds, ranks and head sizes, then the
    first again; each against the workspace backward on its own inputs."""
    big = _near_limit_shape(rfb_lib)
    assert rfb_lib.bwd_workspace_size(*big) > 0.95 * rfb_lib.binding.NOALLOC_SCRATCH_BYTES
    sequence = [(big, 3101), ((2, 3, 64, 32, 8), 3102), ((1, 2, 300, 64, 16), 3103),
                ((1, 1, 129, 64, 0), 3104), (big, 3105)]
    lib = rfb_lib.load_library()
    for call, (shape, seed) in enumerate(sequence, 1):
        g, o, lse, s, ref = _problem(rfb_lib, cuda_dev, shape, seed)
        grads = _nan_grads(g, shape[4])
        rc = _call_noalloc(lib, g, o, lse, grads, shape, s)
        assert rc == 0, rfb_lib.strerror(rc)
        torch.cuda.synchronize()
        assert rfb_lib.last_device_error() == 0
        for name, got, want in zip(("dQ", "dK", "dV", "dU", "dW"), grads, ref):
            if want is None:
                continue
            assert_close(f"call {call} {shape} {name}", got, to_np(want))


def test_noalloc_python_wrapper(rfb_lib, cuda_dev):
    """rank_biased_window_b200.attn_bwd_noalloc on a small problem equals the
    workspace backward; a problem beyond the array raises RuntimeError."""
    shape = (2, 2, 200, 32, 16)
    g, o, lse, s, ref = _problem(rfb_lib, cuda_dev, shape, 3106)
    got = rfb_lib.attn_bwd_noalloc(g["q"], g["k"], g["v"], g["u"], g["w"], o, lse, g["dout"], s)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    for name, a, b in zip(("dQ", "dK", "dV", "dU", "dW"), got, ref):
        assert_close(f"wrapper {name}", a, to_np(b))
    B, H, N, d, r = _near_limit_shape(rfb_lib)
    N += 1024
    t = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device=cuda_dev)
    f = torch.zeros((B, H, N, r), dtype=torch.bfloat16, device=cuda_dev)
    lse2 = torch.zeros((B, H, N), dtype=torch.float32, device=cuda_dev)
    with pytest.raises(RuntimeError, match="fixed"):
        rfb_lib.attn_bwd_noalloc(t, t, t, f, f, t, lse2, t, 0.125)


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
