"""Low-rank factoriser of a materialised bias: the oracle's truncated SVD is
pinned by the Eckart-Young closed form, exact recovery of rank-r input and a
diagonal case; the randomised factoriser's algorithm is checked against the
oracle's optimal error on the CPU (with torch's product standing in for the
library's), and on the GPU with the library's product kernel."""
import numpy as np
import pytest
import torch

import oracle
from rank_biased_window_b200.factorize import _factorize, factorize_bias, relative_position_bias


def _torch_project(B, X, transpose):
    """B X or B^T X with torch: the host-side stand-in for rfb_bias_project,
    so that the factoriser's algorithm can be checked without a GPU."""
    return torch.bmm(B.transpose(1, 2) if transpose else B, X)


def _factorize_cpu(B, r, **kw):
    return _factorize(B, r, _torch_project, **kw)


def test_oracle_error_is_eckart_young():
    """||B - B_r||_F^2 = sum of the eigenvalues of B^T B beyond the r largest
    (eigenvalues from a separate symmetric solver)."""
    rng = np.random.default_rng(5)
    B = rng.standard_normal((3, 20, 20))
    for r in (1, 5, 12):
        _, _, err = oracle.factorize_bias(B, r)
        for h in range(3):
            lam = np.sort(np.linalg.eigvalsh(B[h].T @ B[h]))[::-1]
            want = np.sqrt(lam[r:].sum() / lam.sum())
            assert abs(err[h] - want) < 1e-10


def test_oracle_recovers_exact_low_rank_and_diagonal():
    rng = np.random.default_rng(6)
    U0, W0 = rng.standard_normal((2, 16, 3)), rng.standard_normal((2, 16, 3))
    B = np.einsum("hnr,hmr->hnm", U0, W0)
    U, W, err = oracle.factorize_bias(B, 3)
    np.testing.assert_allclose(np.einsum("hnr,hmr->hnm", U, W), B, atol=1e-10)
    assert err.max() < 1e-12
    d = np.array([5.0, 4.0, 3.0, 2.0, 1.0])
    _, _, err = oracle.factorize_bias(np.diag(d)[None], 2)
    assert abs(err[0] - np.sqrt((d[2:] ** 2).sum() / (d ** 2).sum())) < 1e-14


# Mistakes planted in a copy of the oracle's factoriser must fail its pins.
MUTANTS = [
    ("w_from_left_vectors", "W[h] = Yt[:r].T * root", "W[h] = X[:, :r] * root"),
    ("singular_values_not_split", "root = np.sqrt(S[:r])", "root = S[:r]"),
    ("right_vectors_not_transposed", "W[h] = Yt[:r].T * root", "W[h] = Yt[:, :r] * root"),
]


def _planted(old, new):
    import inspect
    src = inspect.getsource(oracle.factorize_bias)
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<planted>", "exec"), ns)
    return ns["factorize_bias"]


def _pins_hold(fn, monkeypatch):
    monkeypatch.setattr(oracle, "factorize_bias", fn)
    try:
        test_oracle_error_is_eckart_young()
        test_oracle_recovers_exact_low_rank_and_diagonal()
    except AssertionError:
        return False
    return True


def test_oracle_pins_hold_for_the_unmodified_copy(monkeypatch):
    assert _pins_hold(_planted("root = np.sqrt(S[:r])", "root = np.sqrt(S[:r])"), monkeypatch)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_oracle_pins_catch_planted_mistake(name, old, new, monkeypatch):
    assert not _pins_hold(_planted(old, new), monkeypatch), name


@pytest.mark.parametrize("r", [4, 8, 16])
def test_randomised_factoriser_near_optimal_cpu(r):
    B = relative_position_bias(3, 8, 8, seed=11)
    U, W, err = _factorize_cpu(B, r, out_dtype=torch.float32)
    assert U.shape == (3, 64, r) and W.shape == (3, 64, r)
    _, _, opt = oracle.factorize_bias(B.double().numpy(), r)
    # within 2 % of the best possible rank-r error (power iterations converge fast)
    assert (err.numpy() <= opt * 1.02 + 1e-5).all(), (err, opt)
    # reported error matches the factors returned
    R = B - torch.bmm(U, W.transpose(1, 2))
    np.testing.assert_allclose(err.numpy(), (torch.linalg.matrix_norm(R) /
                                             torch.linalg.matrix_norm(B)).numpy(), rtol=1e-4)


def test_randomised_factoriser_exact_rank_and_bf16_output():
    g = torch.Generator().manual_seed(3)
    U0, W0 = torch.randn((2, 48, 8), generator=g), torch.randn((2, 48, 8), generator=g)
    B = torch.bmm(U0, W0.transpose(1, 2))
    U, W, err = _factorize_cpu(B, 8)                       # bf16 factors
    assert U.dtype == torch.bfloat16
    assert err.max().item() < 1e-2                          # bf16 rounding of the factors
    _, _, err32 = _factorize_cpu(B, 8, out_dtype=torch.float32)
    assert err32.max().item() < 1e-5


def test_factoriser_argument_checks():
    with pytest.raises(ValueError):
        _factorize_cpu(torch.zeros(2, 4, 5), 2)
    with pytest.raises(ValueError):
        _factorize_cpu(torch.zeros(2, 4, 4), 0)
    with pytest.raises(ValueError, match="GPU"):      # no CPU path for the public call
        factorize_bias(torch.zeros(2, 4, 4), 2)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(2, 100, 24), (3, 256, 40), (1, 1000, 80), (2, 64, 1)],
                         ids=lambda s: "H{}N{}k{}".format(*s))
def test_bias_project_matches_fp64(rfb_lib, cuda_dev, shape):
    """rfb_bias_project (both orientations) against an fp64 product on the
    host, ragged N included."""
    H, N, k = shape
    g = torch.Generator().manual_seed(N + k)
    B = torch.randn((H, N, N), generator=g)
    X = torch.randn((H, N, k), generator=g)
    for t in (False, True):
        got = rfb_lib.bias_project(B.to(cuda_dev), X.to(cuda_dev), t).double().cpu()
        want = torch.bmm(B.double().transpose(1, 2) if t else B.double(), X.double())
        rel = ((got - want).norm() / want.norm()).item()
        assert rel < 1e-6, (t, rel)


@pytest.mark.gpu
@pytest.mark.parametrize("r", [8, 16, 32])
def test_gpu_factoriser_near_optimal(rfb_lib, cuda_dev, r):
    """The factoriser with the library's products on a 16 x 16-window bias:
    within 2 % of the best possible rank-r error (fp32 factors)."""
    B = relative_position_bias(4, 16, 16, seed=13, device=cuda_dev)
    U, W, err = factorize_bias(B, r, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    _, _, opt = oracle.factorize_bias(B.double().cpu().numpy(), r)
    assert (err.cpu().numpy() <= opt * 1.02 + 1e-5).all(), (err, opt)


@pytest.mark.gpu
def test_factorised_bias_feeds_the_kernels(rfb_lib, cuda_dev):
    """On the GPU: factorise a window bias, then run the factored kernel with
    the factors and the dense comparator with their product U W^T; the two
    compute the same attention (up to bf16 rounding of the product)."""
    from rank_biased_window_b200.inputs import make_inputs
    H, wh, ww, r, B = 4, 16, 16, 32, 3
    bias = relative_position_bias(H, wh, ww, seed=21, device=cuda_dev)
    U, W, err = factorize_bias(bias, r)
    _, _, opt = oracle.factorize_bias(bias.double().cpu().numpy(), r)
    assert (err.cpu().numpy() <= opt * 1.05 + 4e-3).all()   # bf16 factors
    N, d = wh * ww, 32
    x = make_inputs(B, H, N, d, 0, seed=22)
    g = {k: v.to(cuda_dev) for k, v in x.items()}
    o1, _ = rfb_lib.attn_fwd_shared_bias(g["q"], g["k"], g["v"], U, W)
    prod = torch.bmm(U.float(), W.float().transpose(1, 2)).to(torch.bfloat16).contiguous()
    o2, _ = rfb_lib.attn_fwd_dense_bias(g["q"], g["k"], g["v"], prod)
    torch.cuda.synchronize()
    assert rfb_lib.last_device_error() == 0
    diff = (o1.float() - o2.float()).abs().max().item()
    assert diff < 3e-2, diff
