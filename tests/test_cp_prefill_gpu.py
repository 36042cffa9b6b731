"""Context-parallel prefill on one GPU: the ranks are emulated as consecutive
chunks of one sequence.  Rank r computes the partial states of its queries
against its own chunk (causal) and every earlier chunk (in full) with
plx_fwd_partial and merges them with plx_fwd_merge; the ranks' outputs,
concatenated, are compared with plx_fwd over the whole sequence and with the
oracle."""
import pytest
import torch

import oracle
from parity import assert_close
from parameterized_local_linear_plx_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def plx():
    from parameterized_local_linear_plx_b200 import build
    build.build()
    from parameterized_local_linear_plx_b200 import plx as m
    assert torch.cuda.is_available()
    return m


def emulate(plx, q, k, v, r, ranks, causal=True):
    """causal: rank rk merges its own chunk (causal) and the earlier chunks (in
    full), rk + 1 blocks; otherwise every chunk in full, `ranks` blocks."""
    N = q.shape[2]
    C = N // ranks

    def chunk(t, i):
        return t[:, :, i * C:(i + 1) * C].contiguous()

    outs, lses = [], []
    for rk in range(ranks):
        qr = chunk(q, rk)
        rr = None if r is None else chunk(r, rk)
        blocks = rk + 1 if causal else ranks
        parts = torch.stack([plx.plx_fwd_partial(qr, chunk(k, j), chunk(v, j), rr, causal=(causal and j == rk))
                             for j in range(blocks)])
        o, l = plx.plx_fwd_merge(parts)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    return torch.cat(outs, dim=2), torch.cat(lses, dim=2)


def close_to_prefill(plx, out, lse, q, k, v, r, causal=True):
    ref_o, ref_l = plx.plx_fwd(q, k, v, r, causal=causal)
    assert (out.float() - ref_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - ref_l).abs().max().item() <= 1e-4


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_chunks_match_prefill_and_oracle(plx, ranks, d):
    """Chunks of 96 rows: every chunk ends inside a 128-key tile."""
    B, Hq, Hkv, C = 2, 4, 2, 96
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, ranks * C, d, seed=10 * ranks + d, device="cuda")
    out, lse = emulate(plx, q, k, v, r, ranks)
    close_to_prefill(plx, out, lse, q, k, v, r)
    ro, rl = oracle.prefill_effective(q.cpu(), k.cpu(), v.cpu(), r.cpu(), True)
    assert_close(out, ro, lse, rl, f"cp prefill ranks={ranks} d={d}")


@pytest.mark.parametrize("ranks", [2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_noncausal_chunks_match_prefill_and_oracle(plx, ranks, d):
    """Every rank merges all `ranks` chunks in full; chunks of 96 rows."""
    B, Hq, Hkv, C = 2, 4, 2, 96
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, ranks * C, d, seed=70 + 10 * ranks + d, device="cuda")
    out, lse = emulate(plx, q, k, v, r, ranks, causal=False)
    close_to_prefill(plx, out, lse, q, k, v, r, causal=False)
    ro, rl = oracle.prefill_effective(q.cpu(), k.cpu(), v.cpu(), r.cpu(), False)
    assert_close(out, ro, lse, rl, f"cp prefill non-causal ranks={ranks} d={d}")


def test_rho_none_and_odd_group(plx):
    """G = 3 (units of one head) and rho = 0 (the probe branch is zero)."""
    B, Hq, Hkv, d, ranks, C = 1, 3, 1, 128, 3, 200
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, ranks * C, d, seed=5, device="cuda")
    for rr in (None, r):
        out, lse = emulate(plx, q, k, v, rr, ranks)
        close_to_prefill(plx, out, lse, q, k, v, rr)
        ro, rl = oracle.prefill_effective(q.cpu(), k.cpu(), v.cpu(), None if rr is None else rr.cpu(), True)
        assert_close(out, ro, lse, rl, f"cp prefill G=3 rho={'none' if rr is None else 'r'}")


def test_one_full_block_is_the_noncausal_forward(plx):
    """One block over all keys, merged alone, is plx_fwd with causal = 0; its
    records are normalised consistently (lse from m and l)."""
    B, Hq, Hkv, N, d = 2, 4, 4, 300, 64
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=7, device="cuda")
    part = plx.plx_fwd_partial(q, k, v, r, causal=False)
    out, lse = plx.plx_fwd_merge(part[None])
    torch.cuda.synchronize()
    close_to_prefill(plx, out, lse, q, k, v, r, causal=False)
    m, l = part[..., 0], part[..., 1]
    assert torch.isfinite(m).all() and (l > 0).all()
    lse2 = (m + torch.log2(l)) * 0.6931471805599453
    assert (lse2 - lse).abs().max().item() <= 1e-4


def test_bench_shape_four_chunks(plx):
    """Causal prefill B=1, N=4096, Hq=16, Hkv=8, d=128 over 4 emulated ranks."""
    q, k, v, r = inputs.prefill_inputs(1, 16, 8, 4096, 128, seed=0, device="cuda")
    out, lse = emulate(plx, q, k, v, r, 4)
    close_to_prefill(plx, out, lse, q, k, v, r)


def test_context_parallel_prefill_through_nccl_world_one(plx):
    """The full orchestration (all-gather of the key / value chunks, partial
    states, merge) with one rank: it must equal the plain prefill."""
    import datetime
    import socket

    import torch.distributed as dist
    from parameterized_local_linear_plx_b200 import cp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        q, k, v, r = inputs.prefill_inputs(2, 8, 2, 333, 128, seed=12, device="cuda")
        out, lse = cp.context_parallel_prefill(q, k, v, r)
        torch.cuda.synchronize()
        close_to_prefill(plx, out, lse, q, k, v, r)
    finally:
        dist.destroy_process_group()


def emulate_zigzag(plx, q, k, v, r, ranks):
    """Every rank's zig-zag blocks (cp.zigzag_blocks) computed on this GPU from
    chunks of the full tensors, merged per query chunk, then unsharded."""
    from parameterized_local_linear_plx_b200 import cp
    N = q.shape[2]
    c = N // (2 * ranks)

    def chunk(t, i):
        return t[:, :, i * c:(i + 1) * c].contiguous()

    outs, lses = [], []
    for rk in range(ranks):
        local, remote = cp.zigzag_blocks(rk, ranks)
        res = {}
        for qc in cp.zigzag_chunks(rk, ranks):
            blocks = [(kc, causal) for qq, kc, causal in local + remote if qq == qc]
            parts = torch.stack([plx.plx_fwd_partial(chunk(q, qc), chunk(k, kc), chunk(v, kc),
                                                     None if r is None else chunk(r, qc), causal=causal)
                                 for kc, causal in blocks])
            res[qc] = plx.plx_fwd_merge(parts)
        a, b = cp.zigzag_chunks(rk, ranks)
        outs.append(torch.cat([res[a][0], res[b][0]], dim=2))
        lses.append(torch.cat([res[a][1], res[b][1]], dim=2))
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    return cp.zigzag_unshard(outs), cp.zigzag_unshard(lses)


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_zigzag_chunks_match_prefill_and_oracle(plx, ranks, d):
    """Zig-zag layout, chunks of 48 rows (each ends inside a key tile)."""
    B, Hq, Hkv, c = 2, 4, 2, 48
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, 2 * ranks * c, d, seed=90 + 10 * ranks + d, device="cuda")
    out, lse = emulate_zigzag(plx, q, k, v, r, ranks)
    close_to_prefill(plx, out, lse, q, k, v, r)
    ro, rl = oracle.prefill_effective(q.cpu(), k.cpu(), v.cpu(), r.cpu(), True)
    assert_close(out, ro, lse, rl, f"zigzag ranks={ranks} d={d}")


def test_zigzag_bench_shape(plx):
    """Causal prefill B=1, N=4096, Hq=16, Hkv=8, d=128 over 4 emulated ranks
    (8 chunks of 512), rho = 0 and rho."""
    q, k, v, r = inputs.prefill_inputs(1, 16, 8, 4096, 128, seed=3, device="cuda")
    for rr in (None, r):
        out, lse = emulate_zigzag(plx, q, k, v, rr, 4)
        close_to_prefill(plx, out, lse, q, k, v, rr)


def test_zigzag_through_nccl_world_one(plx):
    """The zig-zag orchestration (asynchronous all-gather overlapped by the
    local blocks, remote blocks, two merges) with one rank."""
    import datetime
    import socket

    import torch.distributed as dist
    from parameterized_local_linear_plx_b200 import cp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        q, k, v, r = inputs.prefill_inputs(2, 8, 2, 334, 128, seed=13, device="cuda")
        sh = lambda t: cp.zigzag_shard(t, 0, 1)
        out, lse = cp.context_parallel_prefill_zigzag(sh(q), sh(k), sh(v), sh(r))
        torch.cuda.synchronize()
        out, lse = cp.zigzag_unshard([out]), cp.zigzag_unshard([lse])
        close_to_prefill(plx, out, lse, q, k, v, r)
    finally:
        dist.destroy_process_group()
