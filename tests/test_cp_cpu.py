"""Host side of context parallelism, run as two gloo ranks on the CPU.

Decode: slice planning and the exchange step (the all-gather of partial
states in rank order).  Prefill: the all-gather of the key / value chunks and
the blocks each rank computes (its own chunk causally, every earlier chunk in
full), with the two kernels replaced by fakes that record their calls.  The
kernels themselves are covered by test_cp_decode_gpu.py and
test_cp_prefill_gpu.py."""
import os
import socket
import sys

import torch
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from parameterized_local_linear_plx_b200 import cp
        B, Hq, d = 3, 4, 8
        # a rank's state records, filled with values that name the rank and the position
        part = torch.arange(B * Hq * (2 * d + 4), dtype=torch.float32).reshape(B, Hq, 2 * d + 4)
        part = part + 1000.0 * rank
        g = cp.gather_partials(part)
        q.put((rank, tuple(g.shape), [float(g[i, 0, 0, 0]) for i in range(world)],
               cp.slice_start(rank, 512)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_rank_major():
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
    assert res == [(0, (2, 3, 4, 20), [0.0, 1000.0], 0), (1, (2, 3, 4, 20), [0.0, 1000.0], 512)]


def _worker_prefill(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from parameterized_local_linear_plx_b200 import cp, plx
        calls = []

        def fake_partial(q_, k_, v_, r_=None, causal=True, scale=None, partial=None, stream=None):
            # which chunk this block reads: the chunks are filled with their rank's id
            calls.append((bool(causal), float(k_[0, 0, 0, 0]), float(v_[0, 0, 0, 0]), tuple(partial.shape)))
            partial.fill_(float(k_[0, 0, 0, 0]))
            return partial

        def fake_merge(partials, out=None, lse=None, return_lse=True, stream=None):
            return partials[:, 0, 0, 0, 0].clone(), None

        plx.plx_fwd_partial = fake_partial
        plx.plx_fwd_merge = fake_merge
        B, Hq, Hkv, C, d = 1, 2, 1, 4, 8
        qq = torch.zeros(B, Hq, C, d)
        k = torch.full((B, Hkv, C, d), 10.0 * (rank + 1))
        v = torch.full((B, Hkv, C, d), 100.0 * (rank + 1))
        out, _ = cp.context_parallel_prefill(qq, k, v)
        n_causal = len(calls)
        out_full, _ = cp.context_parallel_prefill(qq, k, v, causal=False)
        q.put((rank, calls[:n_causal], out.tolist(), calls[n_causal:], out_full.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_prefill_blocks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_prefill, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    shape = (1, 2, 4, 2 * 8 + 4)
    full = [(False, 10.0, 100.0, shape), (False, 20.0, 200.0, shape)]
    assert res[0] == (0, [(True, 10.0, 100.0, shape)], [10.0], full, [10.0, 20.0])
    assert res[1] == (1, [(False, 10.0, 100.0, shape), (True, 20.0, 200.0, shape)], [10.0, 20.0], full, [10.0, 20.0])
