"""rank_biased_window_b200 -- attention with an additive rank-factorised bias
(O = softmax(s Q K^T + U W^T) V) as hand-written sm_100a CUDA kernels behind a
C ABI (include/rfb_attn.h), with a thin ctypes binding.

The library is loaded lazily on the first call; importing the package does not
need a GPU.
"""
from .binding import (  # noqa: F401
    LIB_PATH,
    RFBAttention,
    RFBAttentionSharedBias,
    RFBImageWindows,
    allreduce_bias_grads,
    attn_bwd,
    attn_bwd_image_windows,
    attn_bwd_noalloc,
    attn_bwd_noalloc_setup,
    attn_bwd_shared_bias,
    attn_fwd,
    attn_fwd_dense_bias,
    attn_fwd_image_windows,
    attn_fwd_shared_bias,
    bias_project,
    bwd_image_windows_workspace_size,
    bwd_shared_bias_workspace_size,
    bwd_workspace_size,
    debug_set_wait_limit,
    last_device_error,
    load_library,
    profile_enable,
    profile_read,
    rfb_attention,
    rfb_attention_image_windows,
    rfb_attention_shared_bias,
    selftest_wait_timeout,
    strerror,
)
from .factorize import factorize_bias, relative_position_bias  # noqa: F401

__all__ = ["attn_fwd", "attn_bwd", "attn_bwd_noalloc", "attn_bwd_noalloc_setup", "bwd_workspace_size", "rfb_attention", "RFBAttention",
           "attn_fwd_shared_bias", "attn_fwd_dense_bias", "attn_fwd_image_windows", "attn_bwd_image_windows",
           "bwd_image_windows_workspace_size", "attn_bwd_shared_bias", "bwd_shared_bias_workspace_size",
           "rfb_attention_shared_bias", "RFBAttentionSharedBias",
           "rfb_attention_image_windows", "RFBImageWindows", "allreduce_bias_grads",
           "factorize_bias", "relative_position_bias", "bias_project",
           "last_device_error", "selftest_wait_timeout", "debug_set_wait_limit", "load_library", "strerror", "LIB_PATH", "profile_enable", "profile_read"]
