"""Context-parallel decode on one GPU: the ranks are emulated as slices of one
cache (each slice's partial states by plx_decode_partial, stacked in rank
order as the all-gather would, merged by plx_decode_merge)."""
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


def emulate(plx, q, kc, vc, sl, r, ranks, num_splits=0):
    S = kc.shape[2]
    L = S // ranks
    parts = [plx.plx_decode_partial(q, kc[:, :, i * L:(i + 1) * L].contiguous(), vc[:, :, i * L:(i + 1) * L].contiguous(),
                                    sl, r, key_offset=i * L, num_splits=num_splits) for i in range(ranks)]
    out, lse = plx.plx_decode_merge(torch.stack(parts))
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    return out, lse


@pytest.mark.parametrize("ranks", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
def test_slices_match_decode_and_oracle(plx, ranks, d):
    """Ragged lengths: some sequences end inside the first slice, so later
    ranks hold no live key for them (empty partial states)."""
    B, Hq, Hkv, S = 6, 8, 2, 1024
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=ranks + d, device="cuda")
    sl = torch.tensor([1, 100, 300, 700, 1023, 1024], dtype=torch.int32, device="cuda")
    out, lse = emulate(plx, q, kc, vc, sl, r, ranks)
    ref_o, ref_l = plx.plx_decode(q, kc, vc, sl, r)
    assert (out.float() - ref_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - ref_l).abs().max().item() <= 1e-4
    ro, rl = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), sl.cpu())
    assert_close(out, ro, lse, rl, f"cp ranks={ranks} d={d}")


def test_slices_of_many_short_segments(plx):
    """Slices of 128 keys over 8 ranks at B=100 (800 (b, kv head) segments per
    slice): each slice's records come from the segment plan's 8-warp shape,
    with the key offset of its rank; against the plain decode and sampled
    rows of the oracle."""
    B, Hq, Hkv, S, d = 100, 16, 8, 1024, 128
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=31, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(32)
    sl = torch.randint(0, S + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
    sl[0], sl[1], sl[2] = 0, 1, S
    out, lse = emulate(plx, q, kc, vc, sl, r, 8)
    ref_o, ref_l = plx.plx_decode(q, kc, vc, sl, r)
    step = ref_o.float().abs().clamp_min(1.0) * 2.0 ** -7
    assert bool(((out.float() - ref_o.float()).abs() <= step).all())
    live = sl > 0
    assert (lse[live] - ref_l[live]).abs().max().item() <= 1e-4
    pick = [0, 1, 2, 37, 99]
    ro, rl = oracle.decode_effective(q[pick].cpu(), r[pick].cpu(), kc[pick].cpu(), vc[pick].cpu(), sl[pick].cpu())
    assert_close(out[pick], ro, lse[pick], rl, "cp slices of many short segments")


def test_split_counts_empty_rows_and_rho_none(plx):
    B, Hq, Hkv, S, d = 3, 4, 2, 512, 128
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=9, device="cuda")
    sl = torch.tensor([0, 5, 512], dtype=torch.int32, device="cuda")
    for ns in (1, 3):
        out, lse = emulate(plx, q, kc, vc, sl, None, 4, num_splits=ns)
        assert (out[0].float() == 0).all() and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
        ro, rl = oracle.decode_effective(q.cpu(), None, kc.cpu(), vc.cpu(), sl.cpu())
        assert_close(out[1:], ro[1:], lse[1:], rl[1:], f"cp rho=0 splits={ns}")


def test_bench_shape_eight_slices(plx):
    """B=64, context 4096, Hq=16, Hkv=8, d=128 over 8 emulated ranks."""
    q, kc, vc, r, sl = inputs.decode_inputs(64, 16, 8, 4096, 128, seed=0, device="cuda")
    out, lse = emulate(plx, q, kc, vc, sl, r, 8)
    ref_o, ref_l = plx.plx_decode(q, kc, vc, sl, r)
    assert (out.float() - ref_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - ref_l).abs().max().item() <= 1e-4


def test_context_parallel_decode_through_nccl_world_one(plx):
    """The full orchestration (partial, NCCL all-gather, merge) with one rank:
    it must equal the plain decode."""
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
        q, kc, vc, r, sl = inputs.decode_inputs(4, 8, 2, 777, 128, seed=12, seqlens="ragged", device="cuda")
        out, lse = cp.context_parallel_decode(q, kc, vc, sl, r)
        torch.cuda.synchronize()
        ref_o, ref_l = plx.plx_decode(q, kc, vc, sl, r)
        assert (out.float() - ref_o.float()).abs().max().item() <= 1.6e-2
        assert (lse - ref_l).abs().max().item() <= 1e-4
    finally:
        dist.destroy_process_group()
