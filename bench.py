#!/usr/bin/env python3
"""Throughput of the rank-factorised-bias attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {rfb,reference}]
                    [--workload train] [--no-cpu-baseline] [--no-configs]

A step is one pass of the whole hot path -- forward (O, LSE) and backward
(dQ, dK, dV, dU, dW) -- over one batch of the training workload: B=2 images of a
128x128 token map (N=16384), H=8 heads, d=64, bias rank r=32, bf16, seeded
synthetic inputs (rank_biased_window_b200/inputs.py).  The metric is
algorithmic bf16 TFLOP/s of that step (forward 2*BH*N^2*(2d+r) plus backward
2*BH*N^2*(5d+3r) flops, r counted unpadded), with windows/s beside it.

The same JSON line carries, under "configs", the forward-only workloads (one
8x8 window; 1024 SwinIR-style 8x8 windows; 64 windows of 32x32 tokens; a
64x64 map), each timed with CUDA events with L2 flushed before every step,
with its TFLOP/s, windows/s and binding roof (HBM for windows of <= 128
tokens, the bf16 tensor peak otherwise; launch latency for the single
window).

Multi-GPU: every rank runs its own full workload on its own GPU (independent
problems, weak scaling, no data-path collective); the step time is the max over
ranks and `value` counts the work of all ranks.  `--gpus N` without a torchrun
environment re-launches this script under torch.distributed.run with N local
ranks (127.0.0.1).

`--impl reference` times the fp64 CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload; it is a deliberately slow reference, not
a tuned CPU implementation.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "biased-attn fwd+bwd TFLOP/s (bf16) & % of B200 dense-BF16 peak; windows/s"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("rfb", "reference"), default="rfb")
    ap.add_argument("--workload", default="train")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the forward-only workloads reported under 'configs'")
    ap.add_argument("--factorize", action="store_true",
                    help="time the low-rank factoriser of a dense relative-position bias "
                         "(the step before the path) on this workload's window, r = its rank")
    ap.add_argument("--dense-bias", action="store_true",
                    help="materialised-bias comparator: forward with the bias given as a "
                         "dense bf16 [H, N, N] matrix (U[h] W[h]^T), forward only")
    ap.add_argument("--shared-bias", action="store_true",
                    help="one U, W pair per head shared by all windows; with several "
                         "ranks dU, dW are all-reduced (NCCL) inside the step")
    ap.add_argument("--image-windows", action="store_true",
                    help="shifted-window attention on feature maps (SwinIR-sized: 4 maps of "
                         "128 x 128 tokens, 6 heads, d = 32, r = 8, 8 x 8 windows, shift 4), "
                         "forward + backward from the maps")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target wall seconds of the CPU-baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------- work model
def work(wl):
    BH, N, d, r = wl.B * wl.H, wl.N, wl.d, wl.r
    fwd = 2.0 * BH * N * N * (2 * d + r)
    bwd = 2.0 * BH * N * N * (5 * d + 3 * r) if wl.backward else 0.0
    # bytes that must cross HBM once (inputs read, outputs written), bf16 / fp32
    fwd_bytes = BH * N * (2 * (3 * d + 2 * r + d) + 4)
    bwd_bytes = BH * N * (2 * (5 * d + 2 * r) + 12 + 2 * (3 * d + 2 * r)) if wl.backward else 0
    return fwd, bwd, fwd_bytes, bwd_bytes


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_biased_window_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_hash") != kernel_source_hash():
        return None
    return t.get("dram_bytes_per_launch")


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of per-rank float values (identity without a
    process group).  Every rank must call it with the same number of values."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def throughput_tflops(step_flops, world, ms_per_step):
    """Whole-job TFLOP/s: every rank does `step_flops` per step (weak scaling)
    and the step time is the slowest rank's."""
    return step_flops * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------ clock sampling
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - clocks are reported, not required
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                bits = fn(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        busy = [s for s in self.samples] or [0]
        return {"sm_mhz": statistics.median(busy), "sm_min_mhz": min(busy),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------ CPU reference
def cpu_sample(wl, seconds, x64=None):
    """Times the fp64 oracle on a bounded sample of the workload: forward and the
    query-side backward (dQ, dU) of R query rows of head 0 against all N keys,
    with R calibrated so the sample takes about `seconds`.  Returns
    (credited flops, wall seconds, rows, threads)."""
    import oracle
    from rank_biased_window_b200.inputs import to_f64, workload_inputs
    if x64 is None:
        x = workload_inputs(wl, with_dout=True)
        # only head 0 is touched: slice it to keep the conversion cheap
        x64 = {k: to_f64(v[:1, :1].contiguous()) for k, v in x.items()}
    N, d, r = wl.N, wl.d, wl.r
    s = wl.scale

    def run(rows):
        t0 = time.perf_counter()
        oracle.fwd(x64["q"], x64["k"], x64["v"], x64["u"], x64["w"], s, bh_range=(0, 1),
                   rows=rows)
        if wl.backward:
            oracle.bwd_query_rows(x64["q"], x64["k"], x64["v"], x64["u"], x64["w"], x64["dout"],
                                  s, 0, rows)
        return time.perf_counter() - t0

    probe_rows = list(range(min(64, N)))
    t_probe = run(probe_rows)
    R = int(max(16, min(N, len(probe_rows) * seconds / max(t_probe, 1e-6))))
    rows = list(range(R))
    t = run(rows)
    flops = 2.0 * R * N * (2 * d + r)
    if wl.backward:
        flops += 2.0 * R * N * (3 * d + 2 * r)  # recompute S, dP, [dQ | dU]
    return flops, t, R, oracle.max_threads(), x64


def input_bytes(wl, shared=False, dense=False):
    """Bytes of the step's device inputs (Q, K, V, the factors or the dense
    bias, and dO when the step has a backward)."""
    BH = wl.B * wl.H
    n = 3 * BH * wl.N * wl.d * 2
    if dense:
        n += wl.H * wl.N * wl.N * 2
    elif wl.r > 0:
        n += 2 * (wl.H if shared else BH) * wl.N * wl.r * 2
    if wl.backward and not dense:
        n += BH * wl.N * wl.d * 2
    return n


def workload_config(wl, world, *, shared=False, dense=False):
    """The `config` object of the JSON line.  Both arms build it here, so for
    the same workload and rank count the two lines carry identical configs."""
    nbytes = input_bytes(wl, shared, dense)
    return {
        "workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "r": wl.r,
        "global_batch": wl.B * world, "seq_len": wl.N,
        "parallelism": (f"data parallel over windows x{world}, dU/dW all-reduced (NCCL)"
                        if shared and world > 1 else
                        f"replicas x{world}" if world > 1 else "single GPU"),
        "bias": ("dense [H, N, N] bf16 = U[h] W[h]^T (materialised-bias comparator, "
                 "forward only)" if dense else
                 "U, W [H, N, r] shared by all windows" if shared else
                 "U, W [B, H, N, r] per window and head"),
        "l2": (f"inputs exceed L2 ({nbytes / 2**20:.0f} MiB > 126 MiB), no flush"
               if nbytes > L2_BYTES else
               f"inputs {nbytes / 2**20:.0f} MiB fit in L2: before each step a 512 MiB "
               f"write then read flushes L2 (clean lines), outside the timed events"),
        "note": wl.note,
    }


def run_reference(args, wl, rank, world=1):
    if rank != 0:
        return 0
    per_step = max(1.0, 150.0 / max(args.steps + args.warmup, 1))
    flops, t, R, cores, x64 = cpu_sample(wl, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        f_i, t_i, _, _, _ = cpu_sample_fixed(wl, R, x64)
        if i >= args.warmup:
            times.append(t_i)
    t_step = statistics.mean(times) if times else t
    value = flops / t_step / 1e12
    sample = (f"fp64 oracle, head 0 of {wl.B * wl.H}, {R} of {wl.N} query rows against all keys: "
              f"forward" + (" + query-side backward (dQ, dU)" if wl.backward else ""))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world, shared=getattr(args, "shared_bias", False),
                                  dense=getattr(args, "dense_bias", False)),
        "device": "host cores (fp64 oracle, rank 0 only)",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_sample_fixed(wl, R, x64):
    import oracle
    rows = list(range(R))
    t0 = time.perf_counter()
    oracle.fwd(x64["q"], x64["k"], x64["v"], x64["u"], x64["w"], wl.scale, bh_range=(0, 1),
               rows=rows)
    if wl.backward:
        oracle.bwd_query_rows(x64["q"], x64["k"], x64["v"], x64["u"], x64["w"], x64["dout"],
                              wl.scale, 0, rows)
    t = time.perf_counter() - t0
    flops = 2.0 * R * wl.N * (2 * wl.d + wl.r)
    if wl.backward:
        flops += 2.0 * R * wl.N * (3 * wl.d + 2 * wl.r)
    return flops, t, R, None, x64


# ------------------------------------------------------------------ GPU arm
def run_factorize(args, wl, rank):
    """Times rank_biased_window_b200.factorize_bias on a synthetic
    relative-position bias of this workload's window ([H, N, N], square
    windows) at rank r, and reports the relative error against the best
    possible rank-r error (the oracle's truncated SVD)."""
    import math
    import torch
    from rank_biased_window_b200.factorize import factorize_bias, relative_position_bias
    side = int(round(math.sqrt(wl.N)))
    if side * side != wl.N or rank != 0:
        return
    dev = torch.device("cuda", 0)
    bias = relative_position_bias(wl.H, side, side, seed=wl.seed, device=dev)
    for _ in range(max(args.warmup, 3)):
        factorize_bias(bias, wl.r)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        _, _, err = factorize_bias(bias, wl.r)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    line = {"metric": "low-rank factoriser of a dense bias: ms per call", "value": ms,
            "unit": "ms", "higher_is_better": False, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "data": "synthetic smooth relative-position bias",
            "config": {"workload": wl.name, "H": wl.H, "N": wl.N, "r": wl.r,
                       "window": f"{side}x{side}"},
            "rel_err": [round(float(v), 5) for v in err.tolist()]}
    if not args.no_cpu_baseline:
        sys.path.insert(0, ROOT)
        import oracle
        _, _, opt = oracle.factorize_bias(bias.double().cpu().numpy(), wl.r)
        line["oracle_rel_err"] = [round(float(v), 5) for v in opt.tolist()]
    print(json.dumps(line))


def run_image_windows(args, rank):
    """Forward + backward of shifted-window attention read from channels-last
    maps (attn_fwd_image_windows, attn_bwd_image_windows), L2 flushed clean
    before every step; flops as the window workload's (N = 64 per window)."""
    import torch
    import rank_biased_window_b200 as rfb
    if rank != 0:
        return
    B, Hs, Ws, nh, d, r, shift = 4, 128, 128, 6, 32, 8, 4
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cpu")
    g.manual_seed(20260306)
    mk = lambda *shape, std=1.0: (torch.randn(shape, generator=g) * std).to(torch.bfloat16).to(dev)
    q, k, v, do = (mk(B, Hs, Ws, nh, d) for _ in range(4))
    u, w = mk(nh, 64, r, std=r ** -0.5), mk(nh, 64, r, std=r ** -0.5)
    s = d ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty((B, Hs, Ws, nh), dtype=torch.float32, device=dev)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(u),
             torch.empty_like(w))
    ws = torch.empty(rfb.bwd_image_windows_workspace_size(B, Hs, Ws, nh, d, r), dtype=torch.uint8,
                     device=dev)
    fwd = lambda: rfb.attn_fwd_image_windows(q, k, v, u, w, s, shift=shift, out=o, lse=lse)
    bwd = lambda: rfb.attn_bwd_image_windows(q, k, v, u, w, o, lse, do, s, shift=shift,
                                             workspace=ws, grads=grads)
    for _ in range(max(args.warmup, 3)):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    assert rfb.last_device_error() == 0
    flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)
    evs = []
    rfb.profile_read()
    rfb.profile_enable(True)
    for _ in range(args.steps):
        flush.zero_()
        flush_sum.copy_(flush.view(torch.float32).sum())
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        fwd()
        e[1].record()
        bwd()
        e[2].record()
        evs.append(e)
    torch.cuda.synchronize(dev)
    rfb.profile_enable(False)
    prof = rfb.profile_read()
    t_f = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_b = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    BH, N = B * (Hs // 8) * (Ws // 8) * nh, 64
    fl_f = 2.0 * BH * N * N * (2 * d + r)
    fl_b = 2.0 * BH * N * N * (5 * d + 3 * r)
    line = {"metric": "shifted-window attention on maps, fwd+bwd TFLOP/s (bf16)",
            "value": (fl_f + fl_b) / ((t_f + t_b) * 1e-3) / 1e12, "unit": "TFLOP/s",
            "higher_is_better": True, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_f + t_b, "fwd_ms": t_f, "bwd_ms": t_b,
            "windows_per_s": B * (Hs // 8) * (Ws // 8) / ((t_f + t_b) * 1e-3),
            "kernels": {k: {"avg_ms": v[0] / v[1], "launches": v[1]} for k, v in prof.items()
                        if v[1]},
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) maps, N(0,1/r) factors)",
            "config": {"workload": "image windows", "B": B, "img_h": Hs, "img_w": Ws,
                       "heads": nh, "d": d, "r": r, "win": 8, "shift": shift,
                       "l2": "flushed clean before every step"}}
    print(json.dumps(line))


SWEEP = ("tiny", "swinir", "large", "global")


def config_roofline(wl, kernel_ms, peaks):
    """Binding roof of a forward-only workload's kernel: launch latency for a
    single window, HBM for windows of <= 128 tokens, else the bf16 tensor peak
    (burst figure: these kernels run alone, for well under a second)."""
    fl, _, fb, _ = work(wl)
    if wl.B * wl.H == 1:
        return {"bound": "launch", "achieved": kernel_ms * 1e3, "unit": "us per launch",
                "peak": None, "frac": None}
    if wl.N <= 128:
        ach = fb / (kernel_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "peak_kind": f"HBM copy, {peaks['source']}",
                "traffic": ncu_traffic("fwd", wl.name)}
    ach = fl / (kernel_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": ach / peaks["bf16_tflops"], "peak_kind": f"bf16 burst, {peaks['source']}",
            "traffic": ncu_traffic("fwd", wl.name)}


def graph_stream(rfb, torch, dev, wl, g, peaks, dist, world):
    """The same forward issued back to back from one CUDA graph: K launches
    rotating over R copies of the inputs whose total is over 3x L2, so that no
    launch finds its inputs in L2 (L2 also flushed before each replay); one
    pair of events around each replay, time per launch = replay time / K.
    This separates the kernel's throughput from the per-launch latency (a
    few microseconds between consecutive kernels on the device) that the
    per-step events include."""
    fl, _, fb, _ = work(wl)
    R = max(2, -(-3 * L2_BYTES // fb))
    K = max(8, 2 * R)
    sets = []
    for _ in range(R):
        c = {k: v.clone() for k, v in g.items()}
        sets.append((c, torch.empty_like(c["q"]),
                     torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)))

    def launch(i):
        c, o, lse = sets[i % R]
        u, w = (c["u"], c["w"]) if wl.r else (None, None)
        rfb.attn_fwd(c["q"], c["k"], c["v"], u, w, wl.scale, out=o, lse=lse, stream=stream)

    # graphs are captured on a side stream (not the default one)
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    for i in range(R):
        launch(i)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            launch(i)
    flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.zero_()
            flush_sum.copy_(flush.view(torch.float32).sum())
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b) / K)
    del graph
    if rfb.last_device_error() != 0:
        raise RuntimeError(f"device error word set by the {wl.name} graph forwards")
    ts.sort()
    ms = max_over_ranks([ts[len(ts) // 2]], dist, dev)[0]
    res = {"us_per_launch": ms * 1e3, "launches": K, "input_sets": R,
           "input_bytes": R * fb, "windows_per_s": wl.B * world / (ms * 1e-3)}
    if wl.N <= 128:
        ach = fb / (ms * 1e-3) / 1e9
        res.update({"achieved": ach, "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]})
    else:
        ach = fl / (ms * 1e-3) / 1e12
        res.update({"achieved": ach, "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"]})
    return res


def run_configs(rfb, torch, dev, stream, dist, world, peaks, steps, warmup):
    """Forward-only workloads (one 8x8 window, SwinIR-style windows, 32x32
    windows, a 64x64 map): per workload `steps` forwards, each preceded by an
    L2 flush (512 MiB written then read, outside the timed events), timed with
    CUDA events on the launching stream and by the library's per-launch
    events; max over ranks."""
    from rank_biased_window_b200.inputs import WORKLOADS, workload_inputs
    flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)
    out = {}
    for name in SWEEP:
        wl = WORKLOADS[name]
        g = {k: v.to(dev) for k, v in workload_inputs(wl, with_dout=False).items()}
        o = torch.empty_like(g["q"])
        lse = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)
        u, w = (g["u"], g["w"]) if wl.r else (None, None)

        def fwd():
            rfb.attn_fwd(g["q"], g["k"], g["v"], u, w, wl.scale, out=o, lse=lse, stream=stream)

        for _ in range(max(warmup, 3)):
            fwd()
        torch.cuda.synchronize(dev)
        if rfb.last_device_error() != 0:
            raise RuntimeError(f"device error word set by the {name} forward")
        rfb.profile_read()
        rfb.profile_enable(True)
        evs = []
        for _ in range(steps):
            with torch.cuda.stream(stream):
                flush.zero_()
                flush_sum.copy_(flush.view(torch.float32).sum())
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fwd()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        rfb.profile_enable(False)
        prof = rfb.profile_read()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        kms = prof["fwd"][0] / max(prof["fwd"][1], 1)
        ms, kms = max_over_ranks([ms, kms], dist, dev)
        fl, _, fb, _ = work(wl)
        out[name] = {
            "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "r": wl.r, "pass": "fwd",
            "ms_per_step": ms, "kernel_ms": kms,
            "tflops": throughput_tflops(fl, world, ms),
            "kernel_tflops": fl / (kms * 1e-3) / 1e12,
            "windows_per_s": wl.B * world / (ms * 1e-3),
            "pct_of_bf16_peak": fl / (kms * 1e-3) / 1e12 / peaks["bf16_tflops"] * 100.0,
            "algorithmic_bytes": fb,
            "roofline": config_roofline(wl, kms, peaks),
            "steps": steps, "warmup": max(warmup, 3),
            "l2": "flushed (512 MiB write then read) before every step, outside the timed events",
            "note": wl.note,
        }
        if wl.B * wl.H > 1:
            # a supplementary figure: a failure here is recorded, not fatal
            try:
                out[name]["graph_stream"] = graph_stream(rfb, torch, dev, wl, g, peaks, dist,
                                                         world)
            except Exception as e:  # noqa: BLE001
                torch.cuda.synchronize(dev)
                out[name]["graph_stream"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    return out


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_argv(argv, n, port):
    """Command that runs this script under torch.distributed.run with n local
    ranks (one per GPU) on 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.join(ROOT, "bench.py"), *argv]


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # One process per GPU: re-launch under torchrun (rank 0 prints the line).
        import subprocess
        return subprocess.call(relaunch_argv(sys.argv[1:], args.gpus, free_port()))
    from rank_biased_window_b200.inputs import WORKLOADS, workload_inputs
    wl = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; "
                         f"reporting the {world} ranks that run\n")
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    import torch
    import rank_biased_window_b200 as rfb
    from rank_biased_window_b200 import build as rfb_build
    if args.factorize:
        return run_factorize(args, wl, rank)
    if args.image_windows:
        return run_image_windows(args, rank)

    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if rank == 0 and not rfb_build.up_to_date():
        rfb_build.build()
    if dist is not None:
        dist.barrier()
    rfb.load_library()

    x = workload_inputs(wl, with_dout=True)
    shared = (args.shared_bias or args.dense_bias) and wl.r > 0
    dense = args.dense_bias
    if shared:  # one factor pair per head: the first window's
        x["u"], x["w"] = x["u"][0].contiguous(), x["w"][0].contiguous()
    g = {k: v.to(dev) for k, v in x.items()}
    B, H, N, d, r = wl.B, wl.H, wl.N, wl.d, wl.r
    s = wl.scale
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    grads = (torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"]),
             torch.empty_like(g["u"]), torch.empty_like(g["w"]))
    ws_bytes = (rfb.bwd_shared_bias_workspace_size if shared else rfb.bwd_workspace_size)(
        B, H, N, d, r)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    fwd_fn = rfb.attn_fwd_shared_bias if shared else rfb.attn_fwd
    bwd_fn = rfb.attn_bwd_shared_bias if shared else rfb.attn_bwd
    dense_bias = None
    if dense:  # the comparator's input: U[h] W[h]^T materialised once, outside timing
        dense_bias = torch.einsum("hnr,hmr->hnm", g["u"].float(), g["w"].float()).to(
            torch.bfloat16).contiguous()

    def step(gg=None, oo=None, ll=None, gr=None):
        """One step on the device tensors gg -> oo, ll, gr (default: the primary set)."""
        gg = g if gg is None else gg
        oo = o if oo is None else oo
        ll = lse if ll is None else ll
        gr = grads if gr is None else gr
        if dense:
            rfb.attn_fwd_dense_bias(gg["q"], gg["k"], gg["v"], gg.get("bias", dense_bias), s,
                                    out=oo, lse=ll, stream=stream)
            return
        fwd_fn(gg["q"], gg["k"], gg["v"], gg["u"], gg["w"], s, out=oo, lse=ll, stream=stream)
        if wl.backward:
            bwd_fn(gg["q"], gg["k"], gg["v"], gg["u"], gg["w"], oo, ll, gg["dout"], s,
                   workspace=ws, grads=gr, stream=stream)
            if shared and dist is not None:
                # data-parallel windows: the shared factors' gradients are summed
                # over the ranks (the method's one exchange step)
                rfb.allreduce_bias_grads(gr[3], gr[4])

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert rfb.last_device_error() == 0

    # ---- device-timed region: inputs resident in HBM.  When the inputs are
    # larger than L2 the steps run back to back; otherwise L2 is flushed before
    # every step, outside the timed events: a 512 MiB write, then a read of the
    # same buffer so that L2 holds clean lines of other data (a write alone
    # leaves dirty lines whose write-back would be charged to the next step).
    in_bytes = input_bytes(wl, shared, dense)
    flush = None if in_bytes > L2_BYTES else torch.empty(512 * 2**20, dtype=torch.uint8,
                                                        device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)
    rfb.profile_read()
    rfb.profile_enable(True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms_total = e0.elapsed_time(e1)
        else:
            evs = []
            for _ in range(args.steps):
                flush.zero_()
                flush_sum.copy_(flush.view(torch.float32).sum())
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step()
                b.record(stream)
                evs.append((a, b))
            torch.cuda.synchronize(dev)
            ms_total = sum(a.elapsed_time(b) for a, b in evs)
    if dist is not None:
        dist.barrier()
    rfb.profile_enable(False)
    prof = rfb.profile_read()
    err = rfb.last_device_error()
    if err != 0:
        raise RuntimeError(f"device error word {err:#x} after the timed region")

    # ---- end-to-end through the public API with pinned host buffers
    with_grads = wl.backward and not dense
    if dense:  # the comparator's inputs include the dense bias itself
        x["bias"] = dense_bias.cpu()
        g["bias"] = dense_bias
    used = ("q", "k", "v", "bias") if dense else \
        (("q", "k", "v", "u", "w", "dout") if with_grads else ("q", "k", "v", "u", "w"))
    host_in = {k: x[k].pin_memory() for k in used}
    host_out = {"o": torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                "lse": torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)}
    names = ("dq", "dk", "dv", "du", "dw")
    if with_grads:
        for n_, t_ in zip(names, grads):
            host_out[n_] = torch.empty(t_.shape, dtype=t_.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    # Pipelined: every step copies its own inputs in and its results out, but
    # on copy streams, so step k's compute overlaps step k + 1's input copy and
    # step k - 1's read-back (two device buffer sets, ordered by events).
    sets = [(g, o, lse, grads),
            ({k_: torch.empty_like(v_) for k_, v_ in g.items()}, torch.empty_like(o),
             torch.empty_like(lse), tuple(torch.empty_like(t_) for t_ in grads))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(nsteps):
        for kk in range(nsteps):
            b = kk % 2
            gg, oo, ll, gr = sets[b]
            if kk >= 2:
                s_in.wait_event(ev_comp[b])   # step kk - 2 no longer reads these inputs
            with torch.cuda.stream(s_in):
                for k_, v_ in host_in.items():
                    gg[k_].copy_(v_, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if kk >= 2:
                stream.wait_event(ev_out[b])  # step kk - 2's results have been read back
            step(gg, oo, ll, gr)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                host_out["o"].copy_(oo, non_blocking=True)
                host_out["lse"].copy_(ll, non_blocking=True)
                if with_grads:
                    for n_, t_ in zip(names, gr):
                        host_out[n_].copy_(t_, non_blocking=True)
            ev_out[b].record(s_out)

    # as many steps as the device-timed value, so that the first step's input
    # copy and the last step's read-back weigh the same in both
    e2e_steps = max(3, args.steps)
    e2e_run(2)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    e2e_run(e2e_steps)
    stream.wait_event(ev_out[(e2e_steps - 1) % 2])
    f1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e_total = f0.elapsed_time(f1)
    # ---- max over ranks
    ms_total, ms_e2e_total = max_over_ranks([ms_total, ms_e2e_total], dist, dev)

    fwd_f, bwd_f, fwd_b, bwd_b = work(wl)
    if dense:
        # forward only; counted with the factored forward's algorithmic flops for
        # the same attention, so the two lines compare directly
        bwd_f = 0.0
        fwd_b += wl.H * wl.N * wl.N * 2  # the dense bias read once
    step_flops = fwd_f + bwd_f
    ms_step = ms_total / args.steps
    value = throughput_tflops(step_flops, world, ms_step)
    e2e_value = throughput_tflops(step_flops, world, ms_e2e_total / e2e_steps)

    peaks = read_peaks()
    # dominant kernel by measured time
    per = {k: (v[0] / v[1] if v[1] else 0.0, v[1], v[0]) for k, v in prof.items()}
    dom = max(per, key=lambda k: per[k][2])
    dom_flops = {"fwd": fwd_f, "bwd_main": bwd_f}.get(dom)
    launches = sum(v[1] for v in prof.values())
    if dom == "fwd" and wl.N <= 128:
        # Window regime: streaming, HBM-bound (algorithmic bytes per launch).
        achieved = fwd_b / (per[dom][0] * 1e-3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "peak_kind": f"HBM copy, {peaks['source']}", "traffic": ncu_traffic(dom, wl.name),
                "avg_launch_ms": per[dom][0]}
    elif dom_flops is not None:
        # Against the burst bf16 figure (the larger of the two measured peaks,
        # so the lower fraction); the sustained-peak fraction is given beside it.
        achieved = dom_flops / (per[dom][0] * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "peak_kind": f"bf16 burst, {peaks['source']}",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "sustained_peak": peaks["bf16_tflops_sustained"],
                "traffic": ncu_traffic(dom, wl.name),
                "avg_launch_ms": per[dom][0]}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": None, "traffic": None}

    kernels = {k: {"avg_ms": v[0], "launches": v[1], "share": v[2] / max(sum(w[2] for w in
               per.values()), 1e-9)} for k, v in per.items() if v[1]}

    configs = None
    if not args.no_configs:
        configs = run_configs(rfb, torch, dev, stream, dist, world, peaks,
                              max(3, min(args.steps, 20)), args.warmup)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops_c, t_c, R, cores, _ = cpu_sample(wl, args.cpu_seconds)
        cpu = {"value": flops_c / t_c / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"fp64 oracle, head 0 of {wl.B * wl.H}, {R} of {wl.N} query rows "
                         f"against all keys: forward"
                         + (" + query-side backward (dQ, dU)" if wl.backward else "")
                         + f", {t_c:.1f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q,K,V,dO; N(0,1/r) U,W; bf16)",
        "config": workload_config(wl, world, shared=shared, dense=dense),
        "windows_per_s": wl.B * world / (ms_step * 1e-3),
        "pct_of_bf16_peak": value / world / peaks["bf16_tflops"] * 100.0,
        "peaks": peaks,
        "roofline": roof,
        "kernels": kernels,
        "configs": configs,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "note": "every step copies its inputs from pinned host memory and reads its "
                        "results back; the copies run on two copy streams and overlap the "
                        "neighbouring steps' compute"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
