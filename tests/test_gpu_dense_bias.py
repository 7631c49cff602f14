"""GPU parity of the materialised-bias comparator (dense bf16 bias per head)
against the fp64 oracle's dense-bias forward on the same bf16 values."""
import math

import numpy as np
import pytest
import torch

from rank_biased_window_b200.inputs import make_inputs, to_f64
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def _bias(B, H, N, seed, shared):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (H, N, N) if shared else (B, H, N, N)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


CASES = [
    (1, 1, 64, 32, True),
    (2, 2, 200, 64, True),    # ragged last tiles
    (2, 1, 384, 32, False),   # one matrix per window-head
    (1, 3, 136, 64, False),
    (3, 2, 256, 64, True),
]


@pytest.mark.parametrize("shape", CASES, ids=[f"B{b}H{h}N{n}d{d}{'s' if sh else 'w'}"
                                              for b, h, n, d, sh in CASES])
def test_dense_bias_matches_oracle(rfb_lib, oracle_mod, cuda_dev, shape):
    B, H, N, d, shared = shape
    x = make_inputs(B, H, N, d, 0, seed=7000 + N + d)
    bias = _bias(B, H, N, 7100 + N, shared)
    s = 1.0 / math.sqrt(d)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    o, lse = rfb_lib.attn_fwd_dense_bias(g["q"], g["k"], g["v"], bias.to(cuda_dev), s)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    f = {k: to_f64(v) for k, v in x.items()}
    ro, rl = oracle_mod.fwd_dense_bias(f["q"], f["k"], f["v"], to_f64(bias), s)
    assert_close("O", o, ro)
    assert_close("LSE", lse, rl)


def test_dense_bias_of_factors_agrees_with_factored_kernel(rfb_lib, cuda_dev):
    """The comparator fed the materialised U W^T computes the same attention
    as the factored kernel (within bf16 rounding of the bias)."""
    B, H, N, d, r = 2, 2, 512, 64, 32
    x = make_inputs(B, H, N, d, r, seed=7301)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    bias = torch.einsum("bhnr,bhmr->bhnm", g["u"].float(), g["w"].float()).to(torch.bfloat16)
    o1, l1 = rfb_lib.attn_fwd(g["q"], g["k"], g["v"], g["u"], g["w"])
    o2, l2 = rfb_lib.attn_fwd_dense_bias(g["q"], g["k"], g["v"], bias.contiguous())
    assert (o1.float() - o2.float()).abs().max().item() < 3e-2
    assert (l1 - l2).abs().max().item() < 3e-2


def test_dense_bias_rejects_bad_arguments(rfb_lib, cuda_dev):
    x = make_inputs(1, 2, 60, 32, 0, seed=1)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    with pytest.raises(RuntimeError, match="unsupported"):   # N not a multiple of 8
        rfb_lib.attn_fwd_dense_bias(g["q"], g["k"], g["v"],
                                    torch.zeros((2, 60, 60), dtype=torch.bfloat16, device=cuda_dev))
    with pytest.raises(ValueError):
        rfb_lib.attn_fwd_dense_bias(g["q"], g["k"], g["v"],
                                    torch.zeros((3, 60, 60), dtype=torch.bfloat16, device=cuda_dev))
