"""Comparison helpers shared by the GPU parity tests.

Tolerance (per output tensor, against the fp64 oracle on the same bf16 inputs):
max-abs <= 2e-2 and relative L2 (||x - y|| / ||y||) <= 5e-3.
"""
import numpy as np
import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def errors(got, ref):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff)) / nr if nr > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def bf16_floor(ref):
    """Relative L2 error that rounding the exact result to bf16 alone costs."""
    r = np.asarray(ref, dtype=np.float64)
    rb = torch.from_numpy(r).to(torch.bfloat16).to(torch.float64).numpy()
    return errors(rb, r)[1]


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    if isinstance(got, torch.Tensor):
        got = to_np(got)
    if not np.all(np.isfinite(got)):
        raise AssertionError(f"{name}: non-finite values in GPU output")
    ma, rl = errors(got, ref)
    msg = (f"{name}: max-abs {ma:.3e} (<= {max_abs}), rel-L2 {rl:.3e} (<= {rel_l2}), "
           f"bf16 floor {bf16_floor(ref):.2e}")
    assert ma <= max_abs and rl <= rel_l2, msg
    return ma, rl
