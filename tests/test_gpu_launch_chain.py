"""Kernels that read what the kernel just before them wrote, with nothing in
between: the short kernels are launched with programmatic stream
serialisation (each may start while its predecessor finishes and waits for it
with griddepcontrol.wait before touching global memory), so a chain of
dependent launches must give exactly what the same chain gives with a device
synchronisation after every launch, also when the chain is captured into a
CUDA graph and replayed."""
import math

import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _dev(x, dev):
    return {k: v.to(dev) for k, v in x.items()}


def _fwd_chain(rfb, g, s, r, steps, sync):
    """q_{i+1} = O_i: every forward reads the previous forward's output."""
    q = g["q"]
    outs = []
    for _ in range(steps):
        u, w = (g["u"], g["w"]) if r else (None, None)
        o, lse = rfb.attn_fwd(q, g["k"], g["v"], u, w, s)
        if sync:
            torch.cuda.synchronize()
        outs += [o, lse]
        q = o
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("shape", [(300, 1, 64, 32, 8), (2, 3, 640, 64, 16), (4, 6, 49, 32, 0)],
                         ids=["window", "long", "window-ragged"])
def test_dependent_forward_chain_matches_synchronised(rfb_lib, cuda_dev, shape):
    B, H, N, d, r = shape
    g = _dev(make_inputs(B, H, N, d, r, seed=7100 + N), cuda_dev)
    s = 1.0 / math.sqrt(d)
    ref = _fwd_chain(rfb_lib, g, s, r, 6, sync=True)
    got = _fwd_chain(rfb_lib, g, s, r, 6, sync=False)
    assert rfb_lib.last_device_error() == 0
    for i, (a, b) in enumerate(zip(got, ref)):
        assert torch.equal(a, b), f"launch {i // 2} differs"


def _step(rfb, g, s, bufs):
    """forward -> backward -> forward of dQ: each kernel depends on the last."""
    o, lse = rfb.attn_fwd(g["q"], g["k"], g["v"], g["u"], g["w"], s, out=bufs["o"],
                          lse=bufs["lse"])
    rfb.attn_bwd(g["q"], g["k"], g["v"], g["u"], g["w"], o, lse, g["dout"], s,
                 workspace=bufs["ws"], grads=bufs["grads"])
    rfb.attn_fwd(bufs["grads"][0], g["k"], g["v"], g["u"], g["w"], s, out=bufs["o2"],
                 lse=bufs["lse2"])


def _bufs(rfb, g, B, H, N, d, r, dev):
    return {"o": torch.empty_like(g["q"]), "o2": torch.empty_like(g["q"]),
            "lse": torch.empty((B, H, N), dtype=torch.float32, device=dev),
            "lse2": torch.empty((B, H, N), dtype=torch.float32, device=dev),
            "ws": torch.empty(rfb.bwd_workspace_size(B, H, N, d, r), dtype=torch.uint8,
                              device=dev),
            "grads": tuple(torch.empty_like(g[k]) for k in ("q", "k", "v", "u", "w"))}


def _flat(b):
    return [b["o"], b["lse"], *b["grads"], b["o2"], b["lse2"]]


def test_graph_captured_chain_matches_eager(rfb_lib, cuda_dev):
    """Window shapes (N = 64, d = 32, r = 8): forward, window backward and the
    second forward are all deterministic, so the replayed graph must match the
    eager chain bit for bit."""
    B, H, N, d, r = 200, 2, 64, 32, 8
    g = _dev(make_inputs(B, H, N, d, r, seed=7200, with_dout=True), cuda_dev)
    s = 1.0 / math.sqrt(d)
    eager = _bufs(rfb_lib, g, B, H, N, d, r, cuda_dev)
    _step(rfb_lib, g, s, eager)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(cuda_dev)
    side.wait_stream(torch.cuda.current_stream(cuda_dev))
    cap = _bufs(rfb_lib, g, B, H, N, d, r, cuda_dev)
    with torch.cuda.stream(side):
        _step(rfb_lib, g, s, cap)  # warm (descriptors encoded outside the capture)
    torch.cuda.synchronize()
    for t in _flat(cap):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        _step(rfb_lib, g, s, cap)
    for _ in range(2):
        with torch.cuda.stream(side):
            graph.replay()
        torch.cuda.synchronize()
        assert rfb_lib.last_device_error() == 0
        for i, (a, b) in enumerate(zip(_flat(cap), _flat(eager))):
            assert torch.equal(a, b), f"output {i} of the replayed chain differs"
    del graph


def test_concurrent_streams_match_sequential(rfb_lib, cuda_dev):
    """Calls on two streams at once share no device state: a window forward
    and a long forward with its backward (own workspace) on one stream, the
    same on other inputs on a second stream, repeated, give what each gives
    alone.  dQ, dU come from reductions whose order varies and are compared
    with a tolerance of their fp32 rounding; the rest bit for bit."""
    shapes = [(300, 1, 64, 32, 8), (2, 3, 640, 64, 16)]
    sets = []
    for j in range(2):
        for B, H, N, d, r in shapes:
            g = _dev(make_inputs(B, H, N, d, r, seed=7300 + 10 * j + N, with_dout=True), cuda_dev)
            sets.append((g, (B, H, N, d, r), _bufs(rfb_lib, g, B, H, N, d, r, cuda_dev)))

    def run(items, stream):
        with torch.cuda.stream(stream):
            for g, (B, H, N, d, r), b in items:
                s = 1.0 / math.sqrt(d)
                o, lse = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], g["u"], g["w"], s,
                                          out=b["o"], lse=b["lse"])
                rfb_lib.attn_bwd(g["q"], g["k"], g["v"], g["u"], g["w"], o, lse, g["dout"], s,
                                 workspace=b["ws"], grads=b["grads"])

    s0 = torch.cuda.current_stream(cuda_dev)
    run(sets, s0)
    torch.cuda.synchronize()
    ref = [[t.clone() for t in (b["o"], b["lse"], *b["grads"])] for _, _, b in sets]
    sa, sb = torch.cuda.Stream(cuda_dev), torch.cuda.Stream(cuda_dev)
    for _ in range(3):
        for _, _, b in sets:
            for t in (b["o"], b["lse"], *b["grads"]):
                t.zero_()
        torch.cuda.synchronize()
        run(sets[:2] * 2, sa)   # the first input set twice on stream a
        run(sets[2:] * 2, sb)   # the second on stream b, concurrently
        torch.cuda.synchronize()
        assert rfb_lib.last_device_error() == 0
        for (_, shape, b), want in zip(sets, ref):
            got = [b["o"], b["lse"], *b["grads"]]
            for i, (x, y) in enumerate(zip(got, want)):
                if i in (2, 5) and shape[2] > 128:  # dQ, dU of the long backward
                    assert torch.allclose(x.float(), y.float(), rtol=1e-2, atol=1e-3), (shape, i)
                else:
                    assert torch.equal(x, y), (shape, i)
