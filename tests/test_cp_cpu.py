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

import pytest
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


def test_zigzag_layout_round_trip_and_balanced_blocks():
    from parameterized_local_linear_plx_b200 import cp
    for world in (1, 2, 3, 4, 8):
        x = torch.arange(2 * world * 3 * 5, dtype=torch.float32).reshape(1, 1, 2 * world * 3, 5)
        parts = [cp.zigzag_shard(x, rk, world) for rk in range(world)]
        assert torch.equal(cp.zigzag_unshard(parts), x)
        covered = set()
        for rk in range(world):
            local, remote = cp.zigzag_blocks(rk, world)
            blocks = local + remote
            # the same work on every rank: 2 * world + 1 blocks, two of them causal
            assert len(blocks) == 2 * world + 1
            assert sum(1 for _, _, causal in blocks if causal) == 2
            a, b = cp.zigzag_chunks(rk, world)
            for qc, kc, causal in blocks:
                assert qc in (a, b) and kc <= qc and causal == (kc == qc)
                covered.add((qc, kc))
            # the local blocks read only this rank's own chunks
            assert all(kc in (a, b) for _, kc, _ in local)
        # every causal (query chunk, key chunk) pair exactly once over the ranks
        assert covered == {(i, j) for i in range(2 * world) for j in range(i + 1)}
        assert sum(len(sum(cp.zigzag_blocks(rk, world), [])) for rk in range(world)) == len(covered)


def _worker_zigzag(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from parameterized_local_linear_plx_b200 import cp, plx
        calls = []

        def fake_partial(q_, k_, v_, r_=None, causal=True, scale=None, partial=None, stream=None):
            # the chunks are filled with their global chunk id: the block reads (query chunk, key chunk)
            calls.append((int(q_[0, 0, 0, 0]), int(k_[0, 0, 0, 0]), int(v_[0, 0, 0, 0]) - 100, bool(causal)))
            partial.fill_(float(k_[0, 0, 0, 0]))
            return partial

        def fake_merge(partials, out=None, lse=None, return_lse=True, stream=None):
            # out row = the sum of the key chunks merged, as a check of what was merged
            B, Hq, C, pf = partials.shape[1:]
            s = partials[:, :, :, :, :1].sum(0).expand(B, Hq, C, 1).clone()
            return s, torch.zeros(B, Hq, C)

        plx.plx_fwd_partial = fake_partial
        plx.plx_fwd_merge = fake_merge
        B, Hq, Hkv, c, d = 1, 2, 1, 3, 8
        ids = torch.arange(2 * world, dtype=torch.float32).repeat_interleave(c)
        full_q = ids.view(1, 1, -1, 1).expand(B, Hq, 2 * world * c, d).contiguous()
        full_k = ids.view(1, 1, -1, 1).expand(B, Hkv, 2 * world * c, d).contiguous()
        qq = cp.zigzag_shard(full_q, rank, world)
        kk = cp.zigzag_shard(full_k, rank, world)
        vv = cp.zigzag_shard(full_k + 100, rank, world)
        out, _ = cp.context_parallel_prefill_zigzag(qq, kk, vv)
        q.put((rank, calls, out[0, 0, :, 0].tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_zigzag_prefill_blocks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_zigzag, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    from parameterized_local_linear_plx_b200 import cp
    c = 3
    for rank, calls, out in res:
        local, remote = cp.zigzag_blocks(rank, world)
        # every block read the chunk it names (keys and values alike), local blocks first
        assert calls == [(qc, kc, kc, causal) for qc, kc, causal in local + remote]
        a, b = cp.zigzag_chunks(rank, world)
        # the merge of a query chunk saw exactly key chunks 0 .. chunk: their ids sum to chunk (chunk + 1) / 2
        assert out == [a * (a + 1) / 2] * c + [b * (b + 1) / 2] * c
