"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a COPY of the oracle's C source (text
substitution, compiled into a temporary directory) and checks that a library
pin (torch SDPA / autograd in fp64) rejects the planted copy, while the
unmodified copy passes.  Nothing here touches the oracle that the other tests
and the bench use.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from rank_biased_window_b200.inputs import make_inputs, to_f64

# (name, original text, planted text, which pass the mistake lives in)
MUTANTS = [
    ("bias_dropped", "s_row[j] = s * dot(q + i * d, k + j * d, d) + bias_row[j];",
     "s_row[j] = s * dot(q + i * d, k + j * d, d) + 0.0 * bias_row[j];", "fwd"),
    ("bias_transposed", "bias_row[j] = (r > 0) ? dot(u + i * r, w + j * r, r) : 0.0;",
     "bias_row[j] = (r > 0) ? dot(u + j * r, w + i * r, r) : 0.0;", "fwd"),
    ("bias_scaled", "s_row[j] = s * dot(q + i * d, k + j * d, d) + bias_row[j];",
     "s_row[j] = s * (dot(q + i * d, k + j * d, d) + bias_row[j]);", "fwd"),
    ("bias_sign", "s_row[j] = s * dot(q + i * d, k + j * d, d) + bias_row[j];",
     "s_row[j] = s * dot(q + i * d, k + j * d, d) - bias_row[j];", "fwd"),
    ("lse_log2", "return m + log(sum);", "return m + log2(sum);", "fwd"),
    ("ds_sign", "for (long j = 0; j < N; ++j) ds[j] = p[j] * (ds[j] - D);\n                D_all",
     "for (long j = 0; j < N; ++j) ds[j] = p[j] * (D - ds[j]);\n                D_all", "bwd"),
    ("dk_unscaled", "dk[(hh * N + j) * d + c] = s * accK[c];",
     "dk[(hh * N + j) * d + c] = accK[c];", "bwd"),
    ("dw_wrong_operand", "accW[c] += dS * uh[i * r + c];",
     "accW[c] += dS * wh[i * r + c];", "bwd"),
    ("dv_uses_ds", "accV[c] += P * doh[i * d + c];", "accV[c] += dS * doh[i * d + c];", "bwd"),
    ("du_uses_k_side", "for (long j = 0; j < N; ++j) acc += ds[j] * wh[j * r + c];\n"
     "                    du[(hh",
     "for (long j = 0; j < N; ++j) acc += ds[j] * uh[j * r + c];\n                    du[(hh",
     "bwd"),
    ("d_missing", "ds[j] = p[j] * (ds[j] - D);\n                D_all",
     "ds[j] = p[j] * ds[j];\n                D_all", "bwd"),
]


def _inputs():
    t = make_inputs(1, 2, 13, 8, 4, seed=999, with_dout=True)
    return {k: to_f64(v) for k, v in t.items()}


def _fwd_pin_ok(var, x, s):
    o, _ = var.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], s)
    mask = torch.from_numpy(x["u"] @ np.swapaxes(x["w"], -1, -2))
    ref = F.scaled_dot_product_attention(torch.from_numpy(x["q"]), torch.from_numpy(x["k"]),
                                         torch.from_numpy(x["v"]), attn_mask=mask, scale=s)
    sc = (torch.from_numpy(x["q"]) @ torch.from_numpy(x["k"]).transpose(-1, -2) * s + mask)
    _, lse = var.fwd(x["q"], x["k"], x["v"], x["u"], x["w"], s)
    return (np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)
            and np.allclose(lse, torch.logsumexp(sc, -1).numpy(), rtol=0, atol=1e-12))


def _bwd_pin_ok(var, x, s):
    grads = var.bwd(x["q"], x["k"], x["v"], x["u"], x["w"], x["dout"], s)
    t = {k: torch.from_numpy(v.copy()).requires_grad_(True) for k, v in x.items() if k != "dout"}
    o = F.scaled_dot_product_attention(t["q"], t["k"], t["v"],
                                       attn_mask=t["u"] @ t["w"].transpose(-1, -2), scale=s)
    o.backward(torch.from_numpy(x["dout"]))
    return all(np.allclose(g, t[n].grad.numpy(), rtol=0, atol=1e-11)
               for g, n in zip(grads, "qkvuw"))


@pytest.fixture(scope="module")
def source(oracle_mod):
    return oracle_mod.source_text()


def test_unmodified_copy_passes(oracle_mod, source, tmp_path):
    var = oracle_mod.Variant(source, str(tmp_path / "clean"))
    x = _inputs()
    s = 1 / math.sqrt(8)
    assert _fwd_pin_ok(var, x, s)
    assert _bwd_pin_ok(var, x, s)


@pytest.mark.parametrize("name,orig,planted,where", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(oracle_mod, source, tmp_path, name, orig, planted, where):
    assert source.count(orig) >= 1, f"mutation site for {name} not found"
    var = oracle_mod.Variant(source.replace(orig, planted, 1), str(tmp_path / name))
    x = _inputs()
    s = 1 / math.sqrt(8)
    if where == "fwd":
        assert not _fwd_pin_ok(var, x, s), name
    else:
        assert not _bwd_pin_ok(var, x, s), name
