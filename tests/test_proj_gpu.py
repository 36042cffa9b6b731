"""The q/k/v/rho projection kernel on the GPU against the fp64 projection
oracle, through the C ABI: prefill layouts, the decode step with the KV
append fused in (contiguous and paged caches), and the serving step
project -> decode against the attention oracle."""
import numpy as np
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


def make(M, dm, Hq, Hkv, d, seed, with_r=True, device="cuda"):
    """x ~ N(0, 1), W ~ N(0, 1/d_model), bf16: q, k, v of unit scale and, with
    the W_R rows scaled by 0.1, rho ~ 0.1 N(0, 1) as in the input recipe."""
    g = torch.Generator(device=device).manual_seed(seed)
    nout = (2 * Hkv + (2 if with_r else 1) * Hq) * d
    x = torch.randn(M, dm, generator=g, device=device).bfloat16()
    w = torch.randn(nout, dm, generator=g, device=device) / dm ** 0.5
    if with_r:
        w[(Hq + 2 * Hkv) * d:] *= 0.1
    return x, w.bfloat16()


@pytest.mark.parametrize("B,N,dm,Hq,Hkv,d", [
    (2, 200, 1024, 16, 8, 128),   # ragged token count (400 rows: a partial 128-row tile)
    (3, 77, 136, 3, 1, 64),       # d_model not a multiple of 64; head blocks that straddle 256-column tiles
    (1, 1, 64, 2, 2, 128),        # one token
    (2, 130, 512, 4, 1, 128),     # G = 4
])
def test_prefill_projection_matches_oracle(plx, B, N, dm, Hq, Hkv, d):
    x, w = make(B * N, dm, Hq, Hkv, d, seed=B * 100 + N)
    q, k, v, r = plx.plx_qkvr_proj(x, w, B, N, Hq, Hkv, d)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    ref = oracle.qkvr_projection(x.cpu(), w.cpu(), B, N, Hq, Hkv, d)
    for got, want, name in zip((q, k, v, r), ref, "qkvr"):
        assert_close(got, want, what=f"{name} B={B} N={N} dm={dm}", scale_abs=True)


def test_prefill_projection_without_rho_rows(plx):
    """W without W_R: the plain q, k, v projection (softmax attention)."""
    B, N, dm, Hq, Hkv, d = 2, 150, 256, 4, 2, 128
    x, w = make(B * N, dm, Hq, Hkv, d, seed=5, with_r=False)
    q, k, v, r = plx.plx_qkvr_proj(x, w, B, N, Hq, Hkv, d, with_r=False)
    assert r is None
    ref = oracle.qkvr_projection(x.cpu(), w.cpu(), B, N, Hq, Hkv, d, with_r=False)
    for got, want, name in zip((q, k, v), ref[:3], "qkv"):
        assert_close(got, want, what=f"{name} no rho", scale_abs=True)


def test_prefill_projection_full_size_sampled(plx):
    """B=8, N=4096, d_model=1024, Hq=16, Hkv=8, d=128 (the benchmark's
    launch): sampled tokens against the oracle row by row."""
    B, N, dm, Hq, Hkv, d = 8, 4096, 1024, 16, 8, 128
    x, w = make(B * N, dm, Hq, Hkv, d, seed=0)
    q, k, v, r = plx.plx_qkvr_proj(x, w, B, N, Hq, Hkv, d)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    wc = w.cpu()
    for m in [0, 1, 127, 128, 4095, 4096, 17000, B * N - 1]:
        b, t = divmod(m, N)
        rq, rk, rv, rr = oracle.qkvr_projection(x[m:m + 1].cpu(), wc, 1, 1, Hq, Hkv, d)
        for got, want, name in ((q[b, :, t], rq[0, :, 0], "q"), (k[b, :, t], rk[0, :, 0], "k"),
                                (v[b, :, t], rv[0, :, 0], "v"), (r[b, :, t], rr[0, :, 0], "r")):
            assert_close(got, want, what=f"{name} token {m}", scale_abs=True)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_projection_appends_into_the_cache(plx, d):
    B, dm, Hq, Hkv, S = 5, 384, 8, 2, 40
    x, w = make(B, dm, Hq, Hkv, d, seed=7 + d)
    g = torch.Generator(device="cuda").manual_seed(9)
    kc = torch.randn(B, Hkv, S, d, generator=g, device="cuda").bfloat16()
    vc = torch.randn(B, Hkv, S, d, generator=g, device="cuda").bfloat16()
    sl = torch.tensor([0, 10, S - 1, S, -1], dtype=torch.int32, device="cuda")
    kc0, vc0 = kc.clone(), vc.clone()
    q, r, sl_out = plx.plx_qkvr_proj_decode(x, w, kc, vc, sl, Hq)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    rq, rr, rk, rv, rsl = oracle.qkvr_projection_decode(x.cpu(), w.cpu(), kc0.cpu(), vc0.cpu(), sl.cpu(), Hq)
    assert_close(q, rq, what="decode q", scale_abs=True)
    assert_close(r, rr, what="decode r", scale_abs=True)
    assert sl_out.cpu().tolist() == [int(s) for s in rsl] == [1, 11, S, S, -1]
    assert torch.equal(sl.cpu(), torch.tensor([0, 10, S - 1, S, -1], dtype=torch.int32))  # input untouched
    for b, s in enumerate([0, 10, S - 1]):
        assert_close(kc[b, :, s], rk[b, :, s], what=f"k slot b={b}", scale_abs=True)
        assert_close(vc[b, :, s], rv[b, :, s], what=f"v slot b={b}", scale_abs=True)
    # every other row is untouched, bit for bit
    mask = torch.ones(B, S, dtype=torch.bool)
    for b, s in enumerate([0, 10, S - 1]):
        mask[b, s] = False
    mask = mask.cuda()
    assert torch.equal(kc.permute(0, 2, 1, 3)[mask], kc0.permute(0, 2, 1, 3)[mask])
    assert torch.equal(vc.permute(0, 2, 1, 3)[mask], vc0.permute(0, 2, 1, 3)[mask])


def test_decode_projection_paged_equals_contiguous(plx):
    B, dm, Hq, Hkv, d, ps, mp = 4, 256, 4, 2, 128, 16, 5
    x, w = make(B, dm, Hq, Hkv, d, seed=11)
    q0, kp, vp, r0, table, _ = inputs.paged_decode_inputs(B, Hq, Hkv, mp, ps, d, seed=12, device="cuda")
    sl = torch.tensor([0, 17, mp * ps - 1, mp * ps], dtype=torch.int32, device="cuda")
    kc = inputs.gather_pages(kp, table)
    vc = inputs.gather_pages(vp, table)
    qa, ra, sla = plx.plx_qkvr_proj_decode_paged(x, w, kp, vp, table, sl, Hq)
    qb, rb, slb = plx.plx_qkvr_proj_decode(x, w, kc, vc, sl, Hq)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.equal(qa, qb) and torch.equal(ra, rb) and torch.equal(sla, slb)
    assert torch.equal(inputs.gather_pages(kp, table), kc) and torch.equal(inputs.gather_pages(vp, table), vc)


def test_serving_step_project_then_decode(plx):
    """One decode step of a Qwen3-0.6B-shaped layer: project the new tokens
    (k, v appended to the cache), then decode over the lengths the projection
    returns; against the projection oracle followed by the attention oracle."""
    B, dm, Hq, Hkv, d, S = 4, 1024, 16, 8, 128, 300
    x, w = make(B, dm, Hq, Hkv, d, seed=21)
    g = torch.Generator(device="cuda").manual_seed(22)
    kc = torch.randn(B, Hkv, S, d, generator=g, device="cuda").bfloat16()
    vc = torch.randn(B, Hkv, S, d, generator=g, device="cuda").bfloat16()
    sl = torch.tensor([0, 1, 150, 299], dtype=torch.int32, device="cuda")
    kc0, vc0 = kc.cpu(), vc.cpu()
    q, r, sl2 = plx.plx_qkvr_proj_decode(x, w, kc, vc, sl, Hq)
    out, lse = plx.plx_decode(q, kc, vc, sl2, r)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    rq, rr, rk, rv, rsl = oracle.qkvr_projection_decode(x.cpu(), w.cpu(), kc0, vc0, sl.cpu(), Hq)
    # the attention oracle on the oracle's projection, with its q, r, k, v
    # rounded to bf16 as the kernels store them
    bf = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16()
    ro, rl = oracle.decode_effective(bf(rq), bf(rr), bf(rk), bf(rv), torch.tensor(rsl, dtype=torch.int32))
    assert_close(out, ro, lse, rl, "project then decode")
