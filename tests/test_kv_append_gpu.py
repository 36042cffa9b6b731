"""Decode-time KV append (contiguous and paged caches) on the GPU."""
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


@pytest.mark.parametrize("d", [64, 128])
def test_contiguous_append_writes_one_row(plx, d):
    B, Hq, Hkv, S = 5, 4, 2, 96
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=d, device="cuda")
    sl = torch.tensor([0, 17, 95, 96, -1], dtype=torch.int32, device="cuda")  # 96 = full, -1 = invalid
    g = torch.Generator(device="cuda").manual_seed(1)
    kn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    vn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    k0, v0, s0 = kc.clone(), vc.clone(), sl.clone()
    plx.plx_kv_append(kn, vn, kc, vc, sl)
    torch.cuda.synchronize()
    want_k, want_v = k0.clone(), v0.clone()
    for b, pos in enumerate(s0.tolist()):
        if 0 <= pos < S:
            want_k[b, :, pos] = kn[b]
            want_v[b, :, pos] = vn[b]
    assert torch.equal(kc, want_k) and torch.equal(vc, want_v)
    assert sl.tolist() == [1, 18, 96, 96, -1]
    plx.plx_kv_append(kn, vn, kc, vc, sl, advance=False)
    torch.cuda.synchronize()
    assert sl.tolist() == [1, 18, 96, 96, -1]


def test_paged_append_writes_one_row(plx):
    B, Hq, Hkv, ps, mp, d = 4, 4, 2, 16, 6, 128
    q, kp, vp, r, table, _ = inputs.paged_decode_inputs(B, Hq, Hkv, mp, ps, d, seed=3, device="cuda")
    sl = torch.tensor([0, 31, 95, 50], dtype=torch.int32, device="cuda")
    table[3, 50 // ps] = -7  # the slot's page id is invalid: not written
    g = torch.Generator(device="cuda").manual_seed(2)
    kn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    vn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    k0, v0 = kp.clone(), vp.clone()
    plx.plx_kv_append_paged(kn, vn, kp, vp, table, sl)
    torch.cuda.synchronize()
    want_k, want_v = k0.clone(), v0.clone()
    for b, pos in enumerate([0, 31, 95]):
        pg = int(table[b, pos // ps])
        want_k[pg, :, pos % ps] = kn[b]
        want_v[pg, :, pos % ps] = vn[b]
    assert torch.equal(kp, want_k) and torch.equal(vp, want_v)
    assert sl.tolist() == [1, 32, 96, 50]


def test_append_then_decode_attends_the_new_token(plx):
    """One serving step: append this step's k, v, then decode: the query
    attends the old keys and its own."""
    B, Hq, Hkv, S, d = 3, 8, 2, 300, 128
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=5, device="cuda")
    sl = torch.tensor([10, 150, 299], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(4)
    kn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    vn = torch.randn(B, Hkv, d, generator=g, device="cuda").bfloat16()
    plx.plx_kv_append(kn, vn, kc, vc, sl)
    out, lse = plx.plx_decode(q, kc, vc, sl, r)
    torch.cuda.synchronize()
    assert sl.tolist() == [11, 151, 300]
    ro, rl = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), sl.cpu())
    assert_close(out, ro, lse, rl, "append+decode")
