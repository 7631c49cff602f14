"""The C-ABI library builds, loads and exports every symbol its header declares;
host-side argument checks work without a GPU (no compute call is made: every
case here is rejected before anything touches the device)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                names += re.findall(r"RFB_API\s+[\w\s\*]+?\b(rfb_\w+)\s*\(", f.read())
    return names


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for want in ("rfb_attn_fwd", "rfb_attn_bwd", "rfb_attn_bwd_workspace_size", "rfb_strerror",
                 "rfb_last_device_error"):
        assert want in names


def test_library_exports_every_declared_symbol(rfb_lib):
    lib = rfb_lib.load_library()
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    from rank_biased_window_b200.binding import SIGNATURES
    assert set(SIGNATURES) == set(_declared_symbols())


def test_strerror_and_version(rfb_lib):
    lib = rfb_lib.load_library()
    assert lib.rfb_version().decode().startswith("rfb_attn")
    assert "success" in lib.rfb_strerror(0).decode()
    for code in range(1, 7):
        assert lib.rfb_strerror(code).decode() != "unknown status"
    assert lib.rfb_strerror(99).decode() == "unknown status"


def test_host_side_argument_checks(rfb_lib):
    lib = rfb_lib.load_library()
    n = None
    # empty problems are no-ops, whatever the pointers
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 0, 4, 64, 32, 8, 0.1, n) == 0
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 2, 4, 0, 32, 8, 0.1, n) == 0
    # unsupported d / r
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 48, 8, 0.1, n) == 2
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 128, 8, 0.1, n) == 2
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 7, 0.1, n) == 2
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 72, 0.1, n) == 2
    # null pointers, negative sizes, non-finite scale
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, 0.1, n) == 1
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, -1, 1, 64, 32, 8, 0.1, n) == 1
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, float("inf"), n) == 1
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, 0.0, n) == 1
    assert lib.rfb_attn_fwd(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, -0.125, n) == 1
    assert lib.rfb_attn_bwd(*([n] * 14), 0, 1, 1, 64, 32, 8, 0.1, n) == 1


def test_workspace_size(rfb_lib):
    lib = rfb_lib.load_library()
    assert lib.rfb_attn_bwd_workspace_size(0, 1, 64, 32, 8) == 0
    assert lib.rfb_attn_bwd_workspace_size(1, 1, 64, 48, 8) == 0
    B, H, N, d, r = 2, 8, 16384, 64, 32
    ws = lib.rfb_attn_bwd_workspace_size(B, H, N, d, r)
    # the 32-byte rows of bf16 parts of -LSE / s and -D (padded to 128 rows),
    # the fp32 dQ|dU accumulator and the bf16 copy U' = U / s
    need = B * H * N * (d + r) * 4 + B * H * N * 32 + B * H * N * r * 2
    assert need <= ws < need + B * H * 128 * 32 + 1024


def test_shared_bias_host_checks_and_workspace(rfb_lib):
    lib = rfb_lib.load_library()
    n = None
    assert lib.rfb_attn_fwd_shared_bias(n, n, n, n, n, n, n, 0, 4, 64, 32, 8, 0.1, n) == 0
    assert lib.rfb_attn_fwd_shared_bias(n, n, n, n, n, n, n, 1, 1, 64, 32, 7, 0.1, n) == 2
    assert lib.rfb_attn_fwd_shared_bias(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, 0.1, n) == 1
    assert lib.rfb_attn_fwd_shared_bias(n, n, n, n, n, n, n, 1, 1, 64, 32, 8, 0.0, n) == 1
    assert lib.rfb_attn_bwd_shared_bias(*([n] * 6 + [n] + [n] * 7 + [0, 1, 1, 64, 48, 8, 0.1, n])) == 2
    assert lib.rfb_attn_bwd_shared_bias_workspace_size(0, 1, 64, 32, 8) == 0
    B, H, N, d, r = 4, 8, 4096, 64, 32
    ws = lib.rfb_attn_bwd_shared_bias_workspace_size(B, H, N, d, r)
    # as the per-window layout, but U' holds one copy per head (H, not B H)
    # and the per-window fp32 dW is added
    need = (B * H * N * (d + r) * 4 + B * H * N * 32 + H * N * r * 2
            + B * H * N * r * 4)
    assert need <= ws < need + B * H * 128 * 32 + 2048


def test_dense_bias_host_checks(rfb_lib):
    lib = rfb_lib.load_library()
    n = None
    assert lib.rfb_attn_fwd_dense_bias(n, n, n, n, n, n, 0, 2, 64, 32, 2, 0.1, n) == 0
    assert lib.rfb_attn_fwd_dense_bias(n, n, n, n, n, n, 1, 2, 64, 32, 2, 0.1, n) == 1  # nulls
    assert lib.rfb_attn_fwd_dense_bias(n, n, n, n, n, n, 1, 2, 64, 48, 2, 0.1, n) == 2  # d


def test_image_windows_host_checks(rfb_lib):
    lib = rfb_lib.load_library()
    n = None
    f = lib.rfb_attn_fwd_image_windows
    # B, img_h, img_w, heads, d, r, win, shift, scale
    assert f(n, n, n, n, n, n, n, 0, 16, 16, 2, 32, 8, 8, 0, 0.1, n) == 0   # empty
    assert f(n, n, n, n, n, n, n, 1, 16, 16, 2, 32, 8, 16, 0, 0.1, n) == 2  # window 16
    assert f(n, n, n, n, n, n, n, 1, 16, 16, 2, 32, 8, 8, 2, 0.1, n) == 2   # shift 2
    assert f(n, n, n, n, n, n, n, 1, 12, 16, 2, 32, 8, 8, 4, 0.1, n) == 2   # 12 rows
    assert f(n, n, n, n, n, n, n, 1, 16, 16, 2, 48, 8, 8, 4, 0.1, n) == 2   # d
    assert f(n, n, n, n, n, n, n, 1, 16, 16, 2, 32, 8, 8, 4, 0.1, n) == 1   # null pointers
    assert f(n, n, n, n, n, n, n, 1, 16, 16, 2, 32, 8, 8, 4, 0.0, n) == 1   # scale


def test_image_windows_backward_host_checks(rfb_lib):
    lib = rfb_lib.load_library()
    n = None
    f = lib.rfb_attn_bwd_image_windows
    size = lib.rfb_attn_bwd_image_windows_workspace_size
    # 8 pointers, 5 outputs, workspace, bytes, B, img_h, img_w, heads, d, r, win, shift, scale
    args = lambda B, Hs, Ws, d, win, shift, scale, ws=0: (
        [n] * 13 + [n, ws, B, Hs, Ws, 2, d, 8, win, shift, scale, n])
    assert f(*args(0, 16, 16, 32, 8, 0, 0.1)) == 0        # empty
    assert f(*args(1, 16, 16, 32, 16, 0, 0.1)) == 2       # window 16
    assert f(*args(1, 16, 16, 32, 8, 2, 0.1)) == 2        # shift 2
    assert f(*args(1, 12, 16, 32, 8, 4, 0.1)) == 2        # 12 rows
    assert f(*args(1, 16, 16, 48, 8, 4, 0.1)) == 2        # d
    assert f(*args(1, 16, 16, 32, 8, 4, 0.1)) == 1        # null pointers
    assert f(*args(1, 16, 16, 32, 8, 4, 0.0)) == 1        # scale
    # workspace: eight bf16 window tensors, the LSE and the shared-factor backward's
    nwin, heads, d, r = 2 * 2 * 3, 2, 32, 8
    base = lib.rfb_attn_bwd_shared_bias_workspace_size(nwin, heads, 64, d, r)
    t = -(-(nwin * heads * 64 * d * 2) // 256) * 256
    lse = -(-(nwin * heads * 64 * 4) // 256) * 256
    assert size(2, 16, 24, heads, d, r) == 8 * t + lse + base
    assert size(0, 16, 24, heads, d, r) == 0 and size(1, 12, 24, heads, d, r) == 0


def test_binding_rejects_bad_outputs_before_the_library():
    """Output, LSE, gradient and workspace tensors the caller hands in are
    checked on the host (dtype, device, shape, layout) before any pointer
    reaches the kernels."""
    import torch
    from rank_biased_window_b200 import binding as b
    dev = torch.device("cuda", 0)
    lse = torch.zeros(2, 3, dtype=torch.float32)
    with pytest.raises(ValueError, match="must live on"):
        b._check_f32("lse", lse, (2, 3), dev)
    with pytest.raises(TypeError, match="float32"):
        b._check_f32("lse", lse.double(), (2, 3), dev)
    with pytest.raises(ValueError, match="workspace"):
        b._workspace(torch.zeros(64, dtype=torch.uint8), 64, dev)
    q = torch.zeros(1, 2, 16, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must live on"):
        b._grads((q, q, q, None, None), q, None, 0, dev)
    with pytest.raises(TypeError, match="bfloat16"):
        b._grads((q.float(), q, q, None, None), q, None, 0, dev)


def test_bench_accounting_helpers(tmp_path, monkeypatch):
    """bench.py's algorithmic flop / byte counts and the traffic record's
    source-hash gate."""
    import json
    import bench
    from rank_biased_window_b200.inputs import WORKLOADS
    wl = WORKLOADS["train"]
    fwd, bwd, fb, bb = bench.work(wl)
    BH, N, d, r = wl.B * wl.H, wl.N, wl.d, wl.r
    assert fwd == 2.0 * BH * N * N * (2 * d + r)
    assert bwd == 2.0 * BH * N * N * (5 * d + 3 * r)
    assert fb == BH * N * (2 * (3 * d + 2 * r + d) + 4)
    assert bench.work(WORKLOADS["swinir"])[1] == 0.0          # forward-only workload
    assert bench.throughput_tflops(1e12, 2, 1000.0) == 2.0    # weak scaling: all ranks' work
    # a traffic record is used only while the kernel sources are unchanged
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "rank_biased_window_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel one")
    rec = {"source_hash": bench.kernel_source_hash(), "dram_bytes_per_launch": 123.0}
    (tmp_path / "profiles" / "k_w_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("k", "w") == 123.0
    (src / "k.cu").write_text("kernel two")
    assert bench.ncu_traffic("k", "w") is None
    assert bench.ncu_traffic("missing", "w") is None


def test_binding_fails_loudly_without_library(tmp_path):
    from rank_biased_window_b200 import binding
    # a fresh loader pointed at a missing file must raise, never fall back
    saved = binding._lib
    try:
        binding._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved


def test_tmem_io_header_is_the_generators_output():
    """csrc/tmem_io.cuh (the tcgen05.ld / st wrappers) is written by
    csrc/gen_tmem_io.py; the committed header must be exactly its output."""
    import subprocess
    import sys
    gen = os.path.join(ROOT, "rank_biased_window_b200", "csrc", "gen_tmem_io.py")
    assert subprocess.run([sys.executable, gen, "--check"]).returncode == 0


def test_noalloc_scratch_size_matches_header():
    """binding.NOALLOC_SCRATCH_BYTES is the header's RFB_NOALLOC_SCRATCH_BYTES."""
    from rank_biased_window_b200 import binding
    with open(os.path.join(ROOT, "include", "rfb_attn.h")) as f:
        m = re.search(r"#define RFB_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", f.read())
    assert m, "RFB_NOALLOC_SCRATCH_BYTES not found in the header"
    a, b, c = (int(x) for x in m.groups())
    assert binding.NOALLOC_SCRATCH_BYTES == a * b * c


def test_wait_limit_hook_host_checks(rfb_lib):
    """The failure-detection hook validates its site on the host and restores
    the defaults with (0, -1); nothing here touches a GPU."""
    lib = rfb_lib.load_library()
    assert lib.rfb_debug_set_wait_limit(0, 256) == 1
    assert lib.rfb_debug_set_wait_limit(0, -2) == 1
    assert lib.rfb_debug_set_wait_limit(5, 13) == 0
    assert lib.rfb_debug_set_wait_limit(0, -1) == 0


def test_bias_project_host_checks(rfb_lib):
    """Argument checks of the factoriser's product entry point happen on the
    host (nothing is launched)."""
    lib = rfb_lib.load_library()
    n = None
    assert lib.rfb_bias_project(n, n, n, 0, 64, 8, 0, n) == 0     # empty
    assert lib.rfb_bias_project(n, n, n, 2, 64, 0, 0, n) == 1     # k < 1
    assert lib.rfb_bias_project(n, n, n, 2, 64, 81, 0, n) == 2    # k > 80
    assert lib.rfb_bias_project(n, n, n, -1, 64, 8, 0, n) == 1    # negative size
    assert lib.rfb_bias_project(n, n, n, 2, 64, 8, 1, n) == 1     # null pointers
