"""The multi-GPU paths on CPU: two `gloo` ranks exercise bench.py's
cross-rank timing reduction (max over ranks) and the whole-job throughput, the
reference arm's rank > 0 exiting without work, and, for bias factors shared
by all windows, the all-reduce that sums each rank's dU, dW over the ranks
(the one data-path exchange; with per-window factors the ranks' work is
independent)."""
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank * 5.0, 3.0 - rank]          # rank 1 is slower on the first value
        got = bench.max_over_ranks(local, dist, "cpu")
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = dict(q.get(timeout=10) for _ in range(world))
    assert results[0] == results[1] == [15.0, 3.0]


def test_throughput_counts_all_ranks():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    # 4948 GFLOP per step on each of 2 ranks, slowest rank 10 ms per step
    assert abs(bench.throughput_tflops(4948e9, 2, 10.0) - 989.6) < 1e-6
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from rank_biased_window_b200.inputs import WORKLOADS

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A(), WORKLOADS["train"], rank=1) == 0
    assert capsys.readouterr().out == ""


def _dp_worker(rank, world, port, q):
    """Data-parallel windows with shared bias factors: each rank holds half of
    the windows, computes its windows' dU, dW (the fp64 oracle stands in for
    the kernels on CPU) and sums them over the ranks with the package's
    all-reduce helper."""
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from rank_biased_window_b200 import allreduce_bias_grads
    from rank_biased_window_b200.inputs import make_inputs, to_f64
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d, r = 4, 2, 24, 8, 8
        x = make_inputs(B, H, N, d, r, seed=123, with_dout=True)
        f = {k: to_f64(v) for k, v in x.items()}
        u = np.broadcast_to(f["u"][0][None], (B, H, N, r)).copy()   # shared factors
        w = np.broadcast_to(f["w"][0][None], (B, H, N, r)).copy()
        lo, hi = rank * B // world, (rank + 1) * B // world           # this rank's windows
        _, _, _, du, dw = oracle.bwd(f["q"][lo:hi], f["k"][lo:hi], f["v"][lo:hi], u[lo:hi],
                                     w[lo:hi], f["dout"][lo:hi], 0.35)
        du_t = torch.from_numpy(du.sum(axis=0))
        dw_t = torch.from_numpy(dw.sum(axis=0))
        allreduce_bias_grads(du_t, dw_t)
        q.put((rank, du_t.numpy(), dw_t.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shared_bias_gradients_all_reduced_over_two_gloo_ranks():
    import numpy as np
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from rank_biased_window_b200.inputs import make_inputs, to_f64
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, H, N, d, r = 4, 2, 24, 8, 8
    x = make_inputs(B, H, N, d, r, seed=123, with_dout=True)
    f = {k: to_f64(v) for k, v in x.items()}
    u = np.broadcast_to(f["u"][0][None], (B, H, N, r)).copy()
    w = np.broadcast_to(f["w"][0][None], (B, H, N, r)).copy()
    _, _, _, du, dw = oracle.bwd(f["q"], f["k"], f["v"], u, w, f["dout"], 0.35)
    for _, du_r, dw_r in got:   # every rank ends with the sum over all windows
        np.testing.assert_allclose(du_r, du.sum(axis=0), rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(dw_r, dw.sum(axis=0), rtol=1e-5, atol=1e-6)


def test_bench_relaunches_itself_for_several_gpus():
    """`bench.py --gpus 2` outside a torchrun environment starts two local
    ranks under torch.distributed.run (127.0.0.1); run here with the reference
    arm (the oracle on the host, no GPU): rank 0 prints one line that counts
    both ranks, rank 1 exits without work, and the line's config is the one
    the GPU arm builds for the same workload and rank count."""
    import json
    import subprocess
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from rank_biased_window_b200.inputs import WORKLOADS
    argv = ["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"]
    cmd = bench.relaunch_argv(argv, 2, 29999)
    assert cmd[1:5] == ["-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2"]
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-len(argv):] == argv
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", *argv],
                         capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(s) for s in res.stdout.splitlines() if s.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"] == bench.workload_config(WORKLOADS["tiny"], 2)
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]


def test_workload_config_is_shared_by_both_arms():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from rank_biased_window_b200.inputs import WORKLOADS
    c = bench.workload_config(WORKLOADS["train"], 1)
    assert c["global_batch"] == 2 and c["seq_len"] == 16384 and c["parallelism"] == "single GPU"
    assert "no flush" in c["l2"]                       # 160 MiB of inputs > L2
    assert "flush" in bench.workload_config(WORKLOADS["swinir"], 1)["l2"]
    assert bench.input_bytes(WORKLOADS["train"]) == 4 * 16 * 16384 * 64 * 2 + 2 * 16 * 16384 * 32 * 2
    assert bench.workload_config(WORKLOADS["train"], 4)["parallelism"] == "replicas x4"
