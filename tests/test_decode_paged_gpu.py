"""Paged-cache decode (block tables) on the GPU: against the contiguous decode
on the gathered cache (bit-exact) and against the fp64 oracle."""
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


def run_both(plx, q, kp, vp, r, table, sl, num_splits=0):
    kc, vc = inputs.gather_pages(kp, table), inputs.gather_pages(vp, table)
    op, lp = plx.plx_decode_paged(q, kp, vp, table, sl, r, num_splits=num_splits)
    oc, lc = plx.plx_decode(q, kc, vc, sl, r, num_splits=num_splits)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    return op, lp, oc, lc, kc, vc


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_page_sizes_equal_contiguous_and_oracle(plx, page_size, d):
    max_pages = max(1, 700 // page_size)
    q, kp, vp, r, table, sl = inputs.paged_decode_inputs(3, 8, 2, max_pages, page_size, d, seed=page_size + d,
                                                         device="cuda")
    op, lp, oc, lc, kc, vc = run_both(plx, q, kp, vp, r, table, sl)
    assert torch.equal(op, oc) and torch.equal(lp, lc)
    ro, rl = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), sl.cpu())
    assert_close(op, ro, lp, rl, f"paged ps={page_size} d={d}")


def test_split_counts_and_rho_none(plx):
    q, kp, vp, r, table, sl = inputs.paged_decode_inputs(2, 4, 2, 40, 32, 128, seed=7, device="cuda")
    for ns in (1, 3, 7):
        op, lp, oc, lc, _, _ = run_both(plx, q, kp, vp, r, table, sl, num_splits=ns)
        assert torch.equal(op, oc) and torch.equal(lp, lc)
    op, lp, oc, lc, kc, vc = run_both(plx, q, kp, vp, None, table, sl)
    assert torch.equal(op, oc)
    ro, rl = oracle.decode_effective(q.cpu(), None, kc.cpu(), vc.cpu(), sl.cpu())
    assert_close(op, ro, lp, rl, "paged rho=0")


def test_unused_table_entries_are_never_read(plx):
    """Entries of page slots past a sequence's live keys may hold anything
    (here -1 and ids past the pool): the result does not change."""
    page_size, max_pages = 16, 12
    q, kp, vp, r, table, _ = inputs.paged_decode_inputs(3, 4, 2, max_pages, page_size, 64, seed=9, device="cuda")
    sl = torch.tensor([5, 100, 192], dtype=torch.int32, device="cuda")
    ref, lref = plx.plx_decode_paged(q, kp, vp, table, sl, r)
    bad = table.clone()
    bad[0, 1:] = -1
    bad[1, 7:] = 1 << 30
    out, lse = plx.plx_decode_paged(q, kp, vp, bad, sl, r)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.equal(out, ref) and torch.equal(lse, lref)


def test_empty_and_clamped_sequences(plx):
    q, kp, vp, r, table, _ = inputs.paged_decode_inputs(3, 4, 2, 5, 64, 128, seed=11, device="cuda")
    sl = torch.tensor([0, -4, 10_000], dtype=torch.int32, device="cuda")
    out, lse = plx.plx_decode_paged(q, kp, vp, table, sl, r)
    torch.cuda.synchronize()
    assert (out[:2].float() == 0).all() and torch.isinf(lse[:2]).all() and (lse[:2] < 0).all()
    kc, vc = inputs.gather_pages(kp, table), inputs.gather_pages(vp, table)
    ro, rl = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), torch.tensor([0, 0, 320]))
    assert_close(out[2], ro[2], lse[2], rl[2], "clamped")


def test_bench_shape_paged(plx):
    """B=64, context 4096, Hq=16, Hkv=8, d=128, pages of 64 keys (the shape the
    benchmark times): equal to the contiguous decode, sampled rows against the oracle."""
    q, kp, vp, r, table, sl = inputs.paged_decode_inputs(64, 16, 8, 64, 64, 128, seed=0, seqlens="equal",
                                                         device="cuda")
    op, lp, oc, lc, kc, vc = run_both(plx, q, kp, vp, r, table, sl)
    assert torch.equal(op, oc) and torch.equal(lp, lc)
    bs = [0, 17, 63]
    rows = [(i, h) for i in range(len(bs)) for h in (0, 5, 15)]
    ro, rl = oracle.decode_rows_explicit(q[bs].cpu(), r[bs].cpu(), kc[bs].cpu(), vc[bs].cpu(), sl[bs].cpu(), rows)
    go = torch.stack([op[bs[i], h] for i, h in rows])
    gl = torch.stack([lp[bs[i], h] for i, h in rows])
    assert_close(go, ro, gl, rl, "paged bench rows")
