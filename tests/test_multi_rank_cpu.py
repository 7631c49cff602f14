"""The multi-GPU path of bench.py on CPU: two `gloo` ranks exercise the
cross-rank timing reduction (max over ranks) and the whole-job throughput, and
the reference arm's rank > 0 exits without work.  The per-rank work itself is
independent (weak scaling, no data-path collective), so nothing else crosses
ranks."""
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
