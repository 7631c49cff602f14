"""fp64 CPU oracle for attention with an additive rank-factorised bias.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it and shares no code with it.

What it computes (per batch-head, scale ``s``)::

    S   = s * Q @ K.T + U @ W.T        # bias matrix formed explicitly
    P   = softmax(S, axis=-1)
    O   = P @ V
    LSE = log(sum(exp(S), axis=-1))    # natural log

following "FlashBias: Fast Computation of Attention with Bias" (Abstract: a
bias matrix added to the query-key scores) and "Rank-Factorized Implicit Neural
Bias" (Abstract: a low-rank bias U W^T).  The backward is the plain chain rule
through the same definition (see ``rfb_oracle.c``).

The arithmetic of ``fwd`` / ``bwd`` / ``bwd_query_rows`` lives in
``rfb_oracle.c`` (plain C, fp64, OpenMP over output rows); this module compiles
it with gcc and marshals numpy arrays.  Three further definitions are written
here in plain numpy (fp64, one head at a time): ``fwd_dense_bias`` (the bias
as a dense matrix), ``factorize_bias`` (best rank-r factors of a dense bias),
``fwd_image_windows`` (shifted-window attention over feature maps) and
``bwd_image_windows`` (its gradients).

Every function is pinned by ``tests/test_oracle_*.py`` against library special
cases (torch SDPA and autograd in fp64), brute force with ``math.fsum``,
closed forms, invariants and finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rfb_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "librfb_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)


def _compile(src: str, out: str) -> str:
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics kept, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return _compile(_SRC, _LIB_PATH)


def _bind(path: str):
    lib = ctypes.CDLL(path)
    L, D, I = ctypes.c_long, ctypes.c_double, ctypes.c_int
    lib.rfb_oracle_fwd.argtypes = [_dp] * 7 + [L] * 4 + [D, L, L, _lp, L, I]
    lib.rfb_oracle_fwd.restype = I
    lib.rfb_oracle_bwd.argtypes = [_dp] * 12 + [L] * 4 + [D, L, L, I]
    lib.rfb_oracle_bwd.restype = I
    lib.rfb_oracle_bwd_query_rows.argtypes = [_dp] * 9 + [L] * 4 + [D, L, _lp, L, I]
    lib.rfb_oracle_bwd_query_rows.restype = I
    lib.rfb_oracle_max_threads.argtypes = []
    lib.rfb_oracle_max_threads.restype = I
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


class Variant:
    """The same Python API bound to a separately compiled copy of the oracle
    source (used by the mutation tests to plant mistakes in a copy)."""

    def __init__(self, src_text: str, workdir: str):
        os.makedirs(workdir, exist_ok=True)
        src = os.path.join(workdir, "variant.c")
        with open(src, "w") as f:
            f.write(src_text)
        self._lib = _bind(_compile(src, os.path.join(workdir, "libvariant.so")))

    def fwd(self, *a, **kw):
        return fwd(*a, _lib_override=self._lib, **kw)

    def bwd(self, *a, **kw):
        return bwd(*a, _lib_override=self._lib, **kw)


def max_threads() -> int:
    return int(_load().rfb_oracle_max_threads())


def _as_f64(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _shape(q, u):
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = q.shape
    r = 0 if u is None else u.shape[-1]
    return B, H, N, d, r


def _prep(q, k, v, u, w):
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d, r = _shape(q, u)
    if r > 0:
        u, w = _as_f64(u), _as_f64(w)
        if u.shape != (B, H, N, r) or w.shape != (B, H, N, r):
            raise ValueError("U, W must be [B, H, N, r]")
    else:
        u = w = None
    for t in (k, v):
        if t.shape != q.shape:
            raise ValueError("Q, K, V must share [B, H, N, d]")
    return q, k, v, u, w, (B, H, N, d, r)


def fwd(q, k, v, u, w, scale, *, nthreads: int = 0, bh_range=None, rows=None,
        _lib_override=None):
    """Forward.  Returns ``(O, LSE)`` as float64.

    With ``bh_range=(bh0, bh1)`` and/or ``rows`` (query indices) only those
    heads / rows are computed; shapes are then ``[bh1-bh0, len(rows), d]`` and
    ``[bh1-bh0, len(rows)]``.  Without them: ``[B, H, N, d]`` and ``[B, H, N]``.
    """
    q, k, v, u, w, (B, H, N, d, r) = _prep(q, k, v, u, w)
    BH = B * H
    bh0, bh1 = (0, BH) if bh_range is None else bh_range
    if rows is None:
        rows_a, nrows = None, N
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = int(rows_a.size)
    nh = bh1 - bh0
    o = np.empty((nh, nrows, d), dtype=np.float64)
    lse = np.empty((nh, nrows), dtype=np.float64)
    rc = (_lib_override or _load()).rfb_oracle_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o), _ptr(lse), BH, N, d, r,
        float(scale), bh0, bh1,
        None if rows_a is None else rows_a.ctypes.data_as(_lp), nrows, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle fwd failed ({rc})")
    if bh_range is None and rows is None:
        return o.reshape(B, H, N, d), lse.reshape(B, H, N)
    return o, lse


def bwd(q, k, v, u, w, dout, scale, *, nthreads: int = 0, bh_range=None, return_D=False,
        _lib_override=None):
    """Full backward.  Returns ``(dQ, dK, dV, dU, dW)`` (dU, dW are None when r == 0),
    shaped like the inputs, or ``[bh1-bh0, N, c]`` with ``bh_range``."""
    q, k, v, u, w, (B, H, N, d, r) = _prep(q, k, v, u, w)
    dout = _as_f64(dout)
    BH = B * H
    bh0, bh1 = (0, BH) if bh_range is None else bh_range
    nh = bh1 - bh0
    dq = np.empty((nh, N, d))
    dk = np.empty((nh, N, d))
    dv = np.empty((nh, N, d))
    du = np.empty((nh, N, r)) if r else None
    dw = np.empty((nh, N, r)) if r else None
    D = np.empty((nh, N))
    rc = (_lib_override or _load()).rfb_oracle_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(dout), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(du), _ptr(dw), _ptr(D), BH, N, d, r, float(scale), bh0, bh1,
        int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle bwd failed ({rc})")
    out = [dq, dk, dv, du, dw]
    if bh_range is None:
        out = [None if t is None else t.reshape(B, H, N, t.shape[-1]) for t in out]
        D = D.reshape(B, H, N)
    return (tuple(out), D) if return_D else tuple(out)


def bwd_query_rows(q, k, v, u, w, dout, scale, bh, rows, *, nthreads: int = 0):
    """dQ_i, dU_i and D_i for the listed query rows of flat head ``bh``."""
    q, k, v, u, w, (B, H, N, d, r) = _prep(q, k, v, u, w)
    dout = _as_f64(dout)
    rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = int(rows_a.size)
    dq = np.empty((n, d))
    du = np.empty((n, r)) if r else None
    D = np.empty(n)
    rc = _load().rfb_oracle_bwd_query_rows(
        _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(dout), _ptr(dq), _ptr(du),
        _ptr(D), B * H, N, d, r, float(scale), int(bh), rows_a.ctypes.data_as(_lp), n,
        int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle bwd_query_rows failed ({rc})")
    return dq, du, D


def fwd_dense_bias(q, k, v, bias, scale):
    """Forward with the bias given as a dense matrix (the materialised form the
    rank-factorised bias replaces; "FlashBias: Fast Computation of Attention
    with Bias", Abstract).  ``bias`` is ``[H, N, N]`` (one matrix per head,
    used by every window) or ``[B, H, N, N]``.  Per batch-head, in float64::

        S = s * Q @ K.T + Bias;  m = max_j S;  P = exp(S - m) / sum_j exp(S - m)
        O = P @ V;  LSE = m + log(sum_j exp(S - m))

    Returns ``(O, LSE)`` shaped ``[B, H, N, d]`` and ``[B, H, N]``.  Pinned in
    ``tests/test_oracle_dense_bias.py`` against the factored oracle (``fwd``)
    with ``Bias = U W^T``."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    bias = np.asarray(bias, dtype=np.float64)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, d))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            bm = bias[h] if bias.ndim == 3 else bias[b, h]
            S = scale * (q[b, h] @ k[b, h].T) + bm
            m = S.max(axis=1, keepdims=True)
            E = np.exp(S - m)
            l = E.sum(axis=1, keepdims=True)
            O[b, h] = (E @ v[b, h]) / l
            L[b, h] = (m + np.log(l))[:, 0]
    return O, L


def factorize_bias(bias, r):
    """Best rank-r factors of each head's bias matrix (Eckart-Young: the
    truncated SVD), the step that turns a materialised bias into the factored
    form ("FlashBias: Fast Computation of Attention with Bias", Abstract: a
    low-rank bias keeps attention fast).  ``bias`` ``[H, N, N]`` float64.
    With Bias_h = X S Y^T (singular values S descending)::

        U_h = X[:, :r] sqrt(S[:r]),   W_h = Y[:, :r] sqrt(S[:r])

    so U_h W_h^T is the rank-r truncation.  Returns ``(U, W, rel_err)`` with
    ``rel_err[h] = ||Bias_h - U_h W_h^T||_F / ||Bias_h||_F``.  Pinned in
    ``tests/test_factorize.py``."""
    bias = np.asarray(bias, dtype=np.float64)
    H, N, _ = bias.shape
    U = np.empty((H, N, r))
    W = np.empty((H, N, r))
    err = np.empty(H)
    for h in range(H):
        X, S, Yt = np.linalg.svd(bias[h])
        root = np.sqrt(S[:r])
        U[h] = X[:, :r] * root
        W[h] = Yt[:r].T * root
        err[h] = np.linalg.norm(bias[h] - U[h] @ W[h].T) / np.linalg.norm(bias[h])
    return U, W, err


def _shift_regions(n, win, shift):
    """Region id along one axis of the cyclically shifted map (the shifted-window
    mask: positions that were not neighbours before the roll get different ids)."""
    ids = np.zeros(n, dtype=np.int64)
    if shift > 0:
        ids[n - win:n - shift] = 1
        ids[n - shift:] = 2
    return ids


def fwd_image_windows(q, k, v, u, w, scale, win, shift):
    """Shifted-window attention over feature maps, written out step by step
    (the window attention of SR transformers such as SwinIR, with the bias in
    the rank-factorised form of "Rank-Factorized Implicit Neural Bias",
    Abstract).  ``q, k, v`` ``[B, Hs, Ws, heads, d]``; ``u, w`` ``[heads,
    win*win, r]`` indexed by the token's raster position inside its window
    (one pair per head, shared by all windows), or None.

    1. roll the maps by (-shift, -shift) over (Hs, Ws);
    2. cut the rolled maps into win x win windows (raster order);
    3. per window and head: S = s Q K^T + U W^T, with S = -inf between tokens
       whose regions of the rolled map differ (when shift > 0);
       P = softmax(S), O = P V, LSE = log sum exp S;
    4. put every token's O and LSE back at its position before the roll.

    Returns ``(O [B, Hs, Ws, heads, d], LSE [B, Hs, Ws, heads])`` in float64."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hs, Ws, nh, d = q.shape
    qs, ks, vs = (np.roll(x, (-shift, -shift), axis=(1, 2)) for x in (q, k, v))
    ry, rx = _shift_regions(Hs, win, shift), _shift_regions(Ws, win, shift)
    O = np.zeros_like(qs)
    L = np.zeros((B, Hs, Ws, nh))
    N = win * win
    for b in range(B):
        for y0 in range(0, Hs, win):
            for x0 in range(0, Ws, win):
                ys, xs = np.meshgrid(np.arange(y0, y0 + win), np.arange(x0, x0 + win), indexing="ij")
                ys, xs = ys.reshape(-1), xs.reshape(-1)           # raster order in the window
                region = 3 * ry[ys] + rx[xs]
                allowed = region[:, None] == region[None, :]
                for h in range(nh):
                    Qw, Kw, Vw = qs[b, ys, xs, h], ks[b, ys, xs, h], vs[b, ys, xs, h]
                    S = scale * (Qw @ Kw.T)
                    if u is not None:
                        S = S + np.asarray(u, dtype=np.float64)[h] @ np.asarray(w, dtype=np.float64)[h].T
                    S = np.where(allowed, S, -np.inf)
                    m = S.max(axis=1, keepdims=True)
                    E = np.exp(S - m)
                    l = E.sum(axis=1, keepdims=True)
                    O[b, ys, xs, h] = (E @ Vw) / l
                    L[b, ys, xs, h] = (m + np.log(l))[:, 0]
    return (np.roll(O, (shift, shift), axis=(1, 2)), np.roll(L, (shift, shift), axis=(1, 2)))


def bwd_image_windows(q, k, v, u, w, dout, scale, win, shift):
    """Gradients of ``fwd_image_windows`` for an upstream gradient ``dout``
    ``[B, Hs, Ws, heads, d]``, by the chain rule through the same steps.  The
    roll and the window cut only move tokens, so every window's gradients are
    those of its own masked attention, carried back to the tokens' places;
    ``u, w`` are shared by all windows, so their gradients are sums over the
    windows.  Per window and head, with P the masked softmax of step 3 (P = 0
    between regions):

        dP = dO V^T,   D_i = sum_j P_ij dP_ij,   dS = P o (dP - D),
        dQ = s dS K,   dK = s dS^T Q,   dV = P^T dO,
        dU[h] += dS W[h],   dW[h] += dS^T U[h].

    Returns ``(dQ, dK, dV, dU, dW)`` in float64; ``dU, dW`` ``[heads, win*win,
    r]`` or None without factors."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, Hs, Ws, nh, d = q.shape
    qs, ks, vs, dos = (np.roll(x, (-shift, -shift), axis=(1, 2)) for x in (q, k, v, do))
    ry, rx = _shift_regions(Hs, win, shift), _shift_regions(Ws, win, shift)
    dQ, dK, dV = np.zeros_like(qs), np.zeros_like(qs), np.zeros_like(qs)
    uu = None if u is None else np.asarray(u, dtype=np.float64)
    ww = None if w is None else np.asarray(w, dtype=np.float64)
    dU = None if uu is None else np.zeros_like(uu)
    dW = None if ww is None else np.zeros_like(ww)
    for b in range(B):
        for y0 in range(0, Hs, win):
            for x0 in range(0, Ws, win):
                ys, xs = np.meshgrid(np.arange(y0, y0 + win), np.arange(x0, x0 + win), indexing="ij")
                ys, xs = ys.reshape(-1), xs.reshape(-1)           # raster order in the window
                region = 3 * ry[ys] + rx[xs]
                allowed = region[:, None] == region[None, :]
                for h in range(nh):
                    Qw, Kw, Vw = qs[b, ys, xs, h], ks[b, ys, xs, h], vs[b, ys, xs, h]
                    dOw = dos[b, ys, xs, h]
                    S = scale * (Qw @ Kw.T)
                    if uu is not None:
                        S = S + uu[h] @ ww[h].T
                    S = np.where(allowed, S, -np.inf)
                    E = np.exp(S - S.max(axis=1, keepdims=True))
                    P = E / E.sum(axis=1, keepdims=True)
                    dP = dOw @ Vw.T
                    Dv = (P * dP).sum(axis=1, keepdims=True)
                    dS = P * (dP - Dv)
                    dQ[b, ys, xs, h] = scale * (dS @ Kw)
                    dK[b, ys, xs, h] = scale * (dS.T @ Qw)
                    dV[b, ys, xs, h] = P.T @ dOw
                    if uu is not None:
                        dU[h] += dS @ ww[h]
                        dW[h] += dS.T @ uu[h]
    back = lambda x: np.roll(x, (shift, shift), axis=(1, 2))
    return back(dQ), back(dK), back(dV), dU, dW
