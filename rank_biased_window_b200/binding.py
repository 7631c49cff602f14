"""ctypes binding of the C ABI in include/rfb_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``librfb_attn.so``.  torch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails, a
``RuntimeError`` is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librfb_attn.so")

RFB_OK = 0
RFB_ERR_INVALID_ARG = 1
RFB_ERR_UNSUPPORTED = 2
RFB_ERR_ALIGNMENT = 3
RFB_ERR_WORKSPACE = 4
RFB_ERR_CUDA = 5
RFB_ERR_DEVICE_TIMEOUT = 6

# Every symbol the header declares, with (restype, argtypes).
_vp, _fp, _i, _f, _sz = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.c_int,
                         ctypes.c_float, ctypes.c_size_t)
SIGNATURES = {
    "rfb_attn_fwd": (_i, [_vp] * 6 + [_fp] + [_i] * 5 + [_f, _vp]),
    "rfb_attn_bwd_workspace_size": (_sz, [_i] * 5),
    "rfb_attn_bwd": (_i, [_vp] * 6 + [_fp] + [_vp] * 7 + [_sz] + [_i] * 5 + [_f, _vp]),
    "rfb_attn_bwd_noalloc": (_i, [_vp] * 6 + [_fp] + [_vp] * 6 + [_i] * 5 + [_f, _vp]),
    "rfb_attn_fwd_shared_bias": (_i, [_vp] * 6 + [_fp] + [_i] * 5 + [_f, _vp]),
    "rfb_attn_bwd_shared_bias_workspace_size": (_sz, [_i] * 5),
    "rfb_attn_fwd_dense_bias": (_i, [_vp] * 5 + [_fp] + [_i] * 5 + [_f, _vp]),
    "rfb_attn_fwd_image_windows": (_i, [_vp] * 6 + [_fp] + [_i] * 8 + [_f, _vp]),
    "rfb_attn_bwd_image_windows_workspace_size": (_sz, [_i] * 6),
    "rfb_attn_bwd_image_windows": (_i, [_vp] * 6 + [_fp] + [_vp] * 7 + [_sz] + [_i] * 8
                                   + [_f, _vp]),
    "rfb_attn_bwd_shared_bias": (_i, [_vp] * 6 + [_fp] + [_vp] * 7 + [_sz] + [_i] * 5 + [_f, _vp]),
    "rfb_strerror": (ctypes.c_char_p, [_i]),
    "rfb_last_device_error": (_i, []),
    "rfb_last_cuda_error": (_i, [ctypes.POINTER(ctypes.c_int)]),
    "rfb_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "rfb_debug_set_wait_limit": (_i, [ctypes.c_uint, _i]),
    "rfb_bias_project": (_i, [_vp, _vp, _vp] + [_i] * 4 + [_vp]),
    "rfb_selftest_soft_exp2": (_i, [_vp, _vp, _i, _vp]),
    "rfb_profile_enable": (_i, [_i]),
    "rfb_profile_read": (_i, [_fp, ctypes.POINTER(ctypes.c_int)]),
    "rfb_profile_kernel_name": (ctypes.c_char_p, [_i]),
    "rfb_version": (ctypes.c_char_p, []),
}
PROFILE_KERNELS = 4

_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load (once) and return the ctypes handle; raises if the .so is absent."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"CUDA library not built: {path} is missing "
                    "(run `python -m rank_biased_window_b200.build`)")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def strerror(code: int) -> str:
    return load_library().rfb_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != RFB_OK:
        extra = ""
        if rc == RFB_ERR_CUDA:
            site = ctypes.c_int(0)
            code = load_library().rfb_last_cuda_error(ctypes.byref(site))
            extra = f"; CUDA error {code} at site {site.value}"
        raise RuntimeError(f"{what} failed: {strerror(rc)} (status {rc}{extra})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class _on_device:
    """Makes `device` current for the call; a no-op when it already is."""

    def __init__(self, device):
        self.ctx = (None if device.index == torch.cuda.current_device()
                    else torch.cuda.device(device))

    def __enter__(self):
        if self.ctx is not None:
            self.ctx.__enter__()

    def __exit__(self, *exc):
        if self.ctx is not None:
            self.ctx.__exit__(*exc)


def _check_operand(name, t, shape, device):
    # Fast path: one combined test; the detailed messages only on failure.
    if (isinstance(t, torch.Tensor) and t.dtype is torch.bfloat16 and t.device == device
            and t.shape == shape and t.is_contiguous()):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must live on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_f32(name, t, shape, device):
    """fp32 tensors the kernels write or read (LSE): dtype, device, shape,
    contiguity -- a wrong one would hand the kernels a bad pointer."""
    if (isinstance(t, torch.Tensor) and t.dtype is torch.float32 and t.device == device
            and t.shape == shape and t.is_contiguous()):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32, got {t.dtype}")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must live on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    raise ValueError(f"{name} must be contiguous")


def _workspace(workspace, nbytes, device):
    """The caller's workspace (or a new one) and its size in bytes; its size
    is checked by the library (RFB_ERR_WORKSPACE), its device and layout here."""
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
            or workspace.device != device or not workspace.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    return workspace, workspace.numel() * workspace.element_size()


def _grads(grads, q, u, r, device):
    """Gradient outputs: new tensors, or the caller's after checking that each
    has its input's shape, dtype and device."""
    if grads is None:
        return (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                torch.empty_like(u) if r else None, torch.empty_like(u) if r else None)
    dq, dk, dv, du, dw = grads
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_operand(name, t, tuple(q.shape), device)
    if r > 0:
        _check_operand("du", du, tuple(u.shape), device)
        _check_operand("dw", dw, tuple(u.shape), device)
        return dq, dk, dv, du, dw
    return dq, dk, dv, None, None


def _dims(q, u):
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = q.shape
    r = 0 if u is None else int(u.shape[-1])
    return int(B), int(H), int(N), int(d), r


def attn_fwd(q, k, v, u=None, w=None, scale=None, *, out=None, lse=None, stream=None):
    """O, LSE = softmax(s Q K^T + U W^T) V, log-sum-exp rows (fp32)."""
    B, H, N, d, r = _dims(q, u)
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_operand(name, t, (B, H, N, d), dev)
    if r > 0:
        _check_operand("u", u, (B, H, N, r), dev)
        _check_operand("w", w, (B, H, N, r), dev)
    else:
        u = w = None
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check_operand("out", o, (B, H, N, d), dev)
    _check_f32("lse", l, (B, H, N), dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(l.data_ptr()), _fp), B, H, N, d, r, s,
            _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_fwd")
    return o, l


def bwd_workspace_size(B, H, N, d, r) -> int:
    return int(load_library().rfb_attn_bwd_workspace_size(B, H, N, d, r))


def attn_bwd(q, k, v, u, w, o, lse, dout, scale=None, *, workspace=None, grads=None,
             stream=None):
    """dQ, dK, dV, dU, dW of L with dL/dO = dout (dU, dW are None when r == 0)."""
    B, H, N, d, r = _dims(q, u)
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_operand(name, t, (B, H, N, d), dev)
    if r > 0:
        _check_operand("u", u, (B, H, N, r), dev)
        _check_operand("w", w, (B, H, N, r), dev)
    else:
        u = w = None
    _check_f32("lse", lse, (B, H, N), dev)
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    dq, dk, dv, du, dw = _grads(grads, q, u, r, dev)
    nbytes = bwd_workspace_size(B, H, N, d, r)
    workspace, ws_bytes = _workspace(workspace, nbytes, dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(lse.data_ptr()), _fp), _ptr(dout), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(du), _ptr(dw), _ptr(workspace), ws_bytes, B, H, N, d, r, s,
            _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_bwd")
    return dq, dk, dv, du, dw


def attn_fwd_shared_bias(q, k, v, u=None, w=None, scale=None, *, out=None, lse=None,
                         stream=None):
    """Forward with one bias-factor pair per head shared by all windows:
    u, w are [H, N, r]; window-head (b, h) uses u[h], w[h]."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    r = 0 if u is None else int(u.shape[-1])
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_operand(name, t, (B, H, N, d), dev)
    if r > 0:
        _check_operand("u", u, (H, N, r), dev)
        _check_operand("w", w, (H, N, r), dev)
    else:
        u = w = None
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check_operand("out", o, (B, H, N, d), dev)
    _check_f32("lse", l, (B, H, N), dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_fwd_shared_bias(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(l.data_ptr()), _fp), B, H, N, d, r, s,
            _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_fwd_shared_bias")
    return o, l


def attn_fwd_dense_bias(q, k, v, bias, scale=None, *, out=None, lse=None, stream=None):
    """Materialised-bias comparator: O = softmax(s Q K^T + bias) V with a dense
    bf16 bias, [H, N, N] (shared by the windows) or [B, H, N, N]."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_operand(name, t, (B, H, N, d), dev)
    if tuple(bias.shape) == (H, N, N):
        bias_heads = H
    elif tuple(bias.shape) == (B, H, N, N):
        bias_heads = B * H
    else:
        raise ValueError(f"bias must be [H, N, N] or [B, H, N, N], got {tuple(bias.shape)}")
    _check_operand("bias", bias, tuple(bias.shape), dev)
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check_operand("out", o, (B, H, N, d), dev)
    _check_f32("lse", l, (B, H, N), dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_fwd_dense_bias(
            _ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(o),
            ctypes.cast(ctypes.c_void_p(l.data_ptr()), _fp), B, H, N, d, bias_heads, s,
            _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_fwd_dense_bias")
    return o, l


def attn_fwd_image_windows(q, k, v, u=None, w=None, scale=None, *, win=8, shift=0, out=None,
                           lse=None, stream=None):
    """Shifted-window attention from feature maps q, k, v [B, H, W, heads, d]
    with shared factors u, w [heads, win*win, r]: returns O [B, H, W, heads, d]
    and LSE [B, H, W, heads] at the tokens' map positions."""
    if q.dim() != 5:
        raise ValueError("q must be [B, H, W, heads, d]")
    B, Hs, Ws, nh, d = (int(x) for x in q.shape)
    r = 0 if u is None else int(u.shape[-1])
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_operand(name, t, (B, Hs, Ws, nh, d), dev)
    if r > 0:
        _check_operand("u", u, (nh, win * win, r), dev)
        _check_operand("w", w, (nh, win * win, r), dev)
    else:
        u = w = None
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hs, Ws, nh), dtype=torch.float32, device=dev) if lse is None else lse
    _check_operand("out", o, (B, Hs, Ws, nh, d), dev)
    _check_f32("lse", l, (B, Hs, Ws, nh), dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_fwd_image_windows(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(l.data_ptr()), _fp), B, Hs, Ws, nh, d, r, int(win),
            int(shift), s, _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_fwd_image_windows")
    return o, l


def bwd_image_windows_workspace_size(B, img_h, img_w, heads, d, r) -> int:
    return int(load_library().rfb_attn_bwd_image_windows_workspace_size(B, img_h, img_w, heads,
                                                                         d, r))


def attn_bwd_image_windows(q, k, v, u, w, o, lse, dout, scale=None, *, win=8, shift=0,
                           workspace=None, grads=None, stream=None):
    """Backward of attn_fwd_image_windows: dQ, dK, dV [B, H, W, heads, d] at
    the tokens' map positions and dU, dW [heads, win*win, r] summed over all
    windows (None when r == 0)."""
    if q.dim() != 5:
        raise ValueError("q must be [B, H, W, heads, d]")
    B, Hs, Ws, nh, d = (int(x) for x in q.shape)
    r = 0 if u is None else int(u.shape[-1])
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_operand(name, t, (B, Hs, Ws, nh, d), dev)
    if r > 0:
        _check_operand("u", u, (nh, win * win, r), dev)
        _check_operand("w", w, (nh, win * win, r), dev)
    else:
        u = w = None
    _check_f32("lse", lse, (B, Hs, Ws, nh), dev)
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    dq, dk, dv, du, dw = _grads(grads, q, u, r, dev)
    nbytes = bwd_image_windows_workspace_size(B, Hs, Ws, nh, d, r)
    workspace, ws_bytes = _workspace(workspace, nbytes, dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_bwd_image_windows(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(lse.data_ptr()), _fp), _ptr(dout), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(du), _ptr(dw), _ptr(workspace), ws_bytes, B, Hs, Ws, nh, d,
            r, int(win), int(shift), s, _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_bwd_image_windows")
    return dq, dk, dv, du, dw


def bwd_shared_bias_workspace_size(B, H, N, d, r) -> int:
    return int(load_library().rfb_attn_bwd_shared_bias_workspace_size(B, H, N, d, r))


def attn_bwd_shared_bias(q, k, v, u, w, o, lse, dout, scale=None, *, workspace=None, grads=None,
                         stream=None):
    """dQ, dK, dV ([B, H, N, d]) and dU, dW ([H, N, r], summed over the B
    windows) for shared bias factors u, w [H, N, r]."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    r = 0 if u is None else int(u.shape[-1])
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_operand(name, t, (B, H, N, d), dev)
    if r > 0:
        _check_operand("u", u, (H, N, r), dev)
        _check_operand("w", w, (H, N, r), dev)
    else:
        u = w = None
    _check_f32("lse", lse, (B, H, N), dev)
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    dq, dk, dv, du, dw = _grads(grads, q, u, r, dev)
    nbytes = bwd_shared_bias_workspace_size(B, H, N, d, r)
    workspace, ws_bytes = _workspace(workspace, nbytes, dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_bwd_shared_bias(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(lse.data_ptr()), _fp), _ptr(dout), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(du), _ptr(dw), _ptr(workspace), ws_bytes, B, H, N, d, r, s,
            _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_bwd_shared_bias")
    return dq, dk, dv, du, dw


def allreduce_bias_grads(du, dw, group=None):
    """Data-parallel windows with shared bias factors: sum each rank's dU, dW
    (already summed over its own windows) over the ranks of `group`, in fp32,
    in place.  Every rank must call it, with tensors of the same shapes."""
    import torch.distributed as dist
    for t in (du, dw):
        if t is None:
            continue
        acc = t.float()
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
        t.copy_(acc)
    return du, dw


# Size of the library's fixed scratch array (RFB_NOALLOC_SCRATCH_BYTES in
# include/rfb_attn.h; a CPU test checks that the two agree).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def attn_bwd_noalloc_setup(device=None, stream=None):
    """Loads the library's kernels on `device` (which reserves the fixed
    scratch array of rfb_attn_bwd_noalloc there) and caches the array's
    address, by an empty call of that entry point.  Call it before reserving
    the rest of the device's memory or capturing a stream on it."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else \
        torch.device(device)
    with _on_device(dev):
        rc = load_library().rfb_attn_bwd_noalloc(
            None, None, None, None, None, None, None, None, None, None, None, None, None,
            0, 1, 1, 64, 0, 0.125, _stream_ptr(stream, dev))
    _check(rc, "rfb_attn_bwd_noalloc (set-up)")


def attn_bwd_noalloc(q, k, v, u, w, o, lse, dout, scale=None, *, grads=None, stream=None):
    """Backward through rfb_attn_bwd_noalloc: the library uses its own fixed
    32 MiB device scratch instead of a caller workspace (for callers that may
    not allocate device memory while they run).  Problems needing more scratch
    than that raise; concurrent calls on one device must be ordered."""
    B, H, N, d, r = _dims(q, u)
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_operand(name, t, (B, H, N, d), dev)
    if r > 0:
        _check_operand("u", u, (B, H, N, r), dev)
        _check_operand("w", w, (B, H, N, r), dev)
    else:
        u = w = None
    _check_f32("lse", lse, (B, H, N), dev)
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    dq, dk, dv, du, dw = _grads(grads, q, u, r, dev)
    with _on_device(dev):
        rc = load_library().rfb_attn_bwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(w), _ptr(o),
            ctypes.cast(ctypes.c_void_p(lse.data_ptr()), _fp), _ptr(dout), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(du), _ptr(dw), B, H, N, d, r, s, _stream_ptr(stream, dev))
    if rc == RFB_ERR_WORKSPACE:
        raise RuntimeError(
            f"rfb_attn_bwd_noalloc: this problem needs {bwd_workspace_size(B, H, N, d, r)} bytes "
            f"of scratch, more than the library's fixed {NOALLOC_SCRATCH_BYTES} bytes")
    _check(rc, "rfb_attn_bwd_noalloc")
    return dq, dk, dv, du, dw


def last_device_error() -> int:
    """Synchronise the current device, read and clear the kernels' error word."""
    return int(load_library().rfb_last_device_error())


def bias_project(bias, x, transpose=False, *, out=None, stream=None):
    """out[h] = bias[h] @ x[h] (or bias[h]^T @ x[h]) on the GPU, fp32:
    bias [H, N, N], x [H, N, k] with k <= 80 (the factoriser's products)."""
    if bias.dim() != 3 or bias.shape[1] != bias.shape[2]:
        raise ValueError("bias must be [H, N, N]")
    H, N, _ = (int(v) for v in bias.shape)
    if x.dim() != 3 or tuple(x.shape[:2]) != (H, N):
        raise ValueError(f"x must be [{H}, {N}, k]")
    k = int(x.shape[2])
    dev = bias.device
    for name, t in (("bias", bias), ("x", x)):
        if t.dtype != torch.float32 or not t.is_cuda or t.device != dev or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 tensor on {dev}")
    o = torch.empty((H, N, k), dtype=torch.float32, device=dev) if out is None else out
    if (o.dtype != torch.float32 or o.device != dev or tuple(o.shape) != (H, N, k)
            or not o.is_contiguous()):
        raise ValueError(f"out must be a contiguous float32 [{H}, {N}, {k}] tensor on {dev}")
    with _on_device(dev):
        rc = load_library().rfb_bias_project(_ptr(bias), _ptr(x), _ptr(o), H, N, k,
                                            1 if transpose else 0, _stream_ptr(stream, dev))
    _check(rc, "rfb_bias_project")
    return o


def debug_set_wait_limit(limit_us: int = 0, fail_site: int = -1):
    """Test hook: main-loop wait limit of the kernels launched afterwards (0:
    the default 2 s) and a wait site that gives up at once (-1: none).
    Process-wide; debug_set_wait_limit() restores the defaults."""
    _check(load_library().rfb_debug_set_wait_limit(int(limit_us), int(fail_site)),
           "rfb_debug_set_wait_limit")


def selftest_wait_timeout(timeout_us: int = 1000, stream=None, device=None):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        rc = load_library().rfb_selftest_wait_timeout(int(timeout_us), _stream_ptr(stream, dev))
    _check(rc, "rfb_selftest_wait_timeout")


def selftest_soft_exp2(x):
    """2^x through the kernels' software exp2 (device fp32 tensor in, out)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        rc = load_library().rfb_selftest_soft_exp2(_ptr(x), _ptr(y), x.numel(),
                                                    _stream_ptr(None, x.device))
    _check(rc, "rfb_selftest_soft_exp2")
    return y


def profile_enable(on: bool = True):
    load_library().rfb_profile_enable(1 if on else 0)


def profile_read():
    """{kernel name: (total ms, launches)} since the last read (synchronises)."""
    lib = load_library()
    ms = (ctypes.c_float * PROFILE_KERNELS)()
    n = (ctypes.c_int * PROFILE_KERNELS)()
    _check(lib.rfb_profile_read(ms, n), "rfb_profile_read")
    return {lib.rfb_profile_kernel_name(i).decode(): (float(ms[i]), int(n[i]))
            for i in range(PROFILE_KERNELS)}


class RFBAttention(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run the CUDA kernels."""

    @staticmethod
    def forward(ctx, q, k, v, u, w, scale):
        o, lse = attn_fwd(q, k, v, u, w, scale)
        ctx.save_for_backward(q, k, v, u, w, o, lse)
        ctx.scale = scale
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, u, w, o, lse = ctx.saved_tensors
        dq, dk, dv, du, dw = attn_bwd(q, k, v, u, w, o, lse, dout.contiguous(), ctx.scale)
        return dq, dk, dv, du, dw, None


class RFBAttentionSharedBias(torch.autograd.Function):
    """Autograd wrapper for shared factors u, w [H, N, r]."""

    @staticmethod
    def forward(ctx, q, k, v, u, w, scale):
        o, lse = attn_fwd_shared_bias(q, k, v, u, w, scale)
        ctx.save_for_backward(q, k, v, u, w, o, lse)
        ctx.scale = scale
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, u, w, o, lse = ctx.saved_tensors
        dq, dk, dv, du, dw = attn_bwd_shared_bias(q, k, v, u, w, o, lse, dout.contiguous(),
                                                  ctx.scale)
        return dq, dk, dv, du, dw, None


class RFBImageWindows(torch.autograd.Function):
    """Autograd wrapper for shifted-window attention on maps q, k, v [B, H, W,
    heads, d] with shared factors u, w [heads, 64, r]."""

    @staticmethod
    def forward(ctx, q, k, v, u, w, scale, shift):
        o, lse = attn_fwd_image_windows(q, k, v, u, w, scale, shift=shift)
        ctx.save_for_backward(q, k, v, u, w, o, lse)
        ctx.scale, ctx.shift = scale, shift
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, u, w, o, lse = ctx.saved_tensors
        dq, dk, dv, du, dw = attn_bwd_image_windows(q, k, v, u, w, o, lse, dout.contiguous(),
                                                    ctx.scale, shift=ctx.shift)
        return dq, dk, dv, du, dw, None, None


def rfb_attention(q, k, v, u, w, scale=None):
    s = (1.0 / math.sqrt(q.shape[-1])) if scale is None else float(scale)
    return RFBAttention.apply(q, k, v, u, w, s)


def rfb_attention_shared_bias(q, k, v, u, w, scale=None):
    """As rfb_attention with u, w [H, N, r] shared by all windows."""
    s = (1.0 / math.sqrt(q.shape[-1])) if scale is None else float(scale)
    return RFBAttentionSharedBias.apply(q, k, v, u, w, s)


def rfb_attention_image_windows(q, k, v, u, w, scale=None, shift=0):
    """Shifted-window attention (8 x 8 windows, shift 0 or 4) on feature maps,
    differentiable in q, k, v, u, w."""
    s = (1.0 / math.sqrt(q.shape[-1])) if scale is None else float(scale)
    return RFBImageWindows.apply(q, k, v, u, w, s, int(shift))
