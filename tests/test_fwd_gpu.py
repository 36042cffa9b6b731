"""Prefill / full-sequence forward on the GPU against the fp64 oracle, through the C ABI."""
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


def run(plx, B, Hq, Hkv, N, d, causal=True, seed=0, use_r=True, r_scale=0.1):
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=seed, r_scale=r_scale)
    out, lse = plx.plx_fwd(q.cuda(), k.cuda(), v.cuda(), r.cuda() if use_r else None, causal=causal)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    ro, rl = oracle.prefill_effective(q, k, v, r if use_r else None, causal)
    return out, lse, ro, rl


def test_tiny_config_fp32_inputs(plx):
    """B=1, H=1, N=256, d=64, fp32 Q, K, V ~ N(0,1), R = 0.1 N(0,1), seed 0:
    the kernel takes the bf16 rounding of the fp32 draws; the oracle runs on the
    same rounded values (explicit Sigma form), and also the R = 0 case."""
    q, k, v, r = inputs.prefill_inputs(1, 1, 1, 256, 64, seed=0, dtype=torch.float32)
    qb, kb, vb, rb = (t.bfloat16() for t in (q, k, v, r))
    out, lse = plx.plx_fwd(qb.cuda(), kb.cuda(), vb.cuda(), rb.cuda(), causal=True)
    ro, rl = oracle.prefill_explicit(qb, kb, vb, rb, causal=True)
    assert_close(out, ro, lse, rl, "tiny")
    out0, lse0 = plx.plx_fwd(qb.cuda(), kb.cuda(), vb.cuda(), None, causal=True)
    ro0, rl0 = oracle.prefill_explicit(qb, kb, vb, None, causal=True)
    assert_close(out0, ro0, lse0, rl0, "tiny rho=0")
    # the unrounded fp32 problem is within the same tolerance of the bf16 result
    rf, _ = oracle.prefill_explicit(q, k, v, r, causal=True)
    assert np.abs(out.float().cpu().numpy() - rf).max() < 5e-2


@pytest.mark.parametrize("N", [1, 2, 3, 17, 64, 127, 128, 129, 200, 256, 300])
@pytest.mark.parametrize("causal", [True, False])
def test_ragged_lengths(plx, N, causal):
    out, lse, ro, rl = run(plx, 1, 2, 1, N, 64, causal=causal, seed=N)
    assert_close(out, ro, lse, rl, f"N={N} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (2, 1), (4, 2), (3, 1), (6, 2), (16, 8)])
def test_heads_and_head_dims(plx, d, Hq, Hkv):
    out, lse, ro, rl = run(plx, 2, Hq, Hkv, 333, d, seed=Hq * 10 + Hkv)
    assert_close(out, ro, lse, rl, f"d={d} Hq={Hq} Hkv={Hkv}")


def test_non_causal_multi_tile(plx):
    out, lse, ro, rl = run(plx, 2, 4, 2, 700, 128, causal=False, seed=21)
    assert_close(out, ro, lse, rl, "non-causal")


def test_r_none_equals_r_zero_and_sdpa(plx):
    q, k, v, r = inputs.prefill_inputs(1, 4, 2, 300, 128, seed=22)
    a = plx.plx_fwd(q.cuda(), k.cuda(), v.cuda(), None)
    b = plx.plx_fwd(q.cuda(), k.cuda(), v.cuda(), torch.zeros_like(r).cuda())
    assert torch.equal(a[0], b[0])
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double().repeat_interleave(2, 1), v.double().repeat_interleave(2, 1), is_causal=True)
    assert (a[0].double().cpu() - ref).abs().max().item() < 1e-2


def test_stress_inputs(plx):
    """Peaked scores (q x 4), correlated values and a large probe (rho ~ N(0,1))."""
    B, Hq, Hkv, N, d = 1, 2, 1, 512, 128
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=23, r_scale=1.0)
    q = (q.float() * 4).bfloat16()
    g = torch.Generator().manual_seed(24)
    W = torch.randn(d, d, generator=g) / d ** 0.5
    v = (k.float() @ W + 0.1 * torch.randn(k.shape, generator=g)).bfloat16()
    out, lse = plx.plx_fwd(q.cuda(), k.cuda(), v.cuda(), r.cuda())
    ro, rl = oracle.prefill_effective(q, k, v, r, True)
    assert_close(out, ro, lse, rl, "stress", scale_abs=True)


def test_decode_row_equals_last_prefill_row(plx):
    B, Hq, Hkv, N, d = 2, 4, 2, 257, 128
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=25)
    out, lse = plx.plx_fwd(q.cuda(), k.cuda(), v.cuda(), r.cuda())
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    od, ld = plx.plx_decode(q[:, :, -1].contiguous().cuda(), k.cuda(), v.cuda(), sl, r[:, :, -1].contiguous().cuda())
    assert (od.float() - out[:, :, -1].float()).abs().max().item() <= 1.6e-2
    assert (ld - lse[:, :, -1]).abs().max().item() <= 1e-3


def test_pretraining_shape_full_size(plx):
    """B=8, N=4096, Hq=16, Hkv=8, d=128, causal, R ~ N(0, 0.1^2): the launch
    the benchmark times.  Sampled rows by the explicit-Sigma oracle (first,
    last, tile edges, random) and two whole heads by the effective form."""
    B, Hq, Hkv, N, d = 8, 16, 8, 4096, 128
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=0, device="cuda")
    out, lse = plx.plx_fwd(q, k, v, r, causal=True)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(0)
    rows = [(0, 0, 0), (0, 0, 1), (7, 15, N - 1), (3, 5, 63), (3, 5, 64), (3, 6, 127), (3, 6, 128),
            (1, 2, 2047), (1, 3, 2048)] + [tuple(int(x) for x in (rng.integers(B), rng.integers(Hq), rng.integers(N)))
                                           for _ in range(40)]
    bs = sorted({rw[0] for rw in rows})
    qc, kc, vc, rc = (t[bs].cpu() for t in (q, k, v, r))
    idx = {bb: i for i, bb in enumerate(bs)}
    ro, rl = oracle.prefill_rows_explicit(qc, kc, vc, rc, [(idx[bb], h, i) for bb, h, i in rows], causal=True)
    go = torch.stack([out[bb, h, i] for bb, h, i in rows])
    gl = torch.stack([lse[bb, h, i] for bb, h, i in rows])
    assert_close(go, ro, gl, rl, "sampled rows")
    for bb, h in [(0, 1), (6, 10)]:
        eo, el = oracle.prefill_effective(q[bb:bb + 1].cpu(), k[bb:bb + 1].cpu(), v[bb:bb + 1].cpu(),
                                          r[bb:bb + 1].cpu(), True, heads=[(0, h)])
        assert_close(out[bb, h], eo[0, h], lse[bb, h], el[0, h], f"head ({bb},{h})")
