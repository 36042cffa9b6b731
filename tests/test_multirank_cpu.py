"""Host-side logic of the multi-GPU benchmark path, run as two gloo ranks on
the CPU: the max-over-ranks timing reduction, the barrier, and the reference
arm's rank-0-only rule.  (The data path has no collective: each rank runs its
own replica of the workload.)"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w, r, lr = bench.dist_setup()
        assert (w, r, lr) == (world, rank, rank)
        t = 10.0 + 5.0 * rank  # each rank's "elapsed ms"
        mx = bench.max_over_ranks(t, world)
        bench.barrier(world)

        class A:
            steps, warmup, gpus = 3, 3, world
        rc = bench.run_reference(A, world, rank) if rank != 0 else 0  # non-zero ranks exit without work
        q.put((rank, mx, rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_barrier():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert res == [(0, 15.0, 0), (1, 15.0, 0)]


def test_single_rank_shortcuts():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_work_counts():
    """The algorithmic byte and flop counts of the benchmark's workloads."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.decode_bytes(64, 16, 8, 128, [4096] * 64) == 64 * 4096 * 8 * 512 + 3 * 64 * 16 * 256 + 4 * 64 * 16
    assert abs(bench.decode_bytes(64, 16, 8, 128, [4096] * 64) / 1e9 - 1.0745) < 1e-3
    assert abs(bench.prefill_flops(8, 16, 4096, 128) / 1e12 - 1.0998) < 1e-3
    assert bench.prefill_flops(1, 1, 3, 2, causal=False) == 8 * 2 * 9
    assert bench.decode_flops(16, 128, [4096] * 64) == 8 * 128 * 16 * 4096 * 64


def test_traffic_figures_only_for_the_captured_sources(monkeypatch):
    """The DRAM traffic in the bench line comes from profiles/ncu_traffic.json
    only while the kernel's source files hash to the captured value."""
    sys.path.insert(0, ROOT)
    import bench
    keys = ("prefill", "decode", "backward")
    for k in keys:
        v = bench.load_traffic(k)
        assert v is None or v > 0
    monkeypatch.setattr(bench, "source_hash", lambda k: "0" * 16)
    assert all(bench.load_traffic(k) is None for k in keys)


def test_backward_flop_count():
    """16d per causal pair: twice the forward's 8d."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.backward_flops(8, 16, 4096, 128) == 2 * bench.prefill_flops(8, 16, 4096, 128)
    assert bench.backward_flops(1, 1, 3, 2, causal=False) == 16 * 2 * 9
