"""Variable-length packed prefill on the GPU: each sequence equals plx_fwd on
that sequence alone (bit for bit) and the fp64 oracle."""
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


def packed_inputs(lens, Hq, Hkv, d, seed, r_scale=0.1):
    """Token-major packed tensors: one fixed-length draw of the longest length,
    each sequence taking its own prefix of a different batch entry."""
    B, N = len(lens), max(lens)
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=seed, r_scale=r_scale, device="cuda")
    pack = lambda t: torch.cat([t[b, :, :n].transpose(0, 1) for b, n in enumerate(lens)]).contiguous()
    cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0)), dtype=torch.int32, device="cuda")
    return pack(q), pack(k), pack(v), pack(r), cu


def check(plx, lens, Hq, Hkv, d, causal, seed, use_r=True, oracle_seqs=()):
    q, k, v, r, cu = packed_inputs(lens, Hq, Hkv, d, seed)
    r = r if use_r else None
    out, lse = plx.plx_fwd_varlen(q, k, v, cu, max(lens), r, causal=causal)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    c = cu.tolist()
    for b, n in enumerate(lens):
        sl = slice(c[b], c[b + 1])
        one = lambda t: t[sl].transpose(0, 1).unsqueeze(0).contiguous()
        o1, l1 = plx.plx_fwd(one(q), one(k), one(v), None if r is None else one(r), causal=causal)
        assert torch.equal(out[sl].transpose(0, 1), o1[0]), f"seq {b} out"
        assert torch.equal(lse[:, sl], l1[0]), f"seq {b} lse"
        if b in oracle_seqs:
            ro, rl = oracle.prefill_effective(one(q).cpu(), one(k).cpu(), one(v).cpu(),
                                              None if r is None else one(r).cpu(), causal)
            assert_close(o1[0], ro[0], l1[0], rl[0], f"seq {b} n={n}")


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_mixed_lengths_pair_heads(plx, causal, d):
    check(plx, [1, 63, 64, 65, 200, 129, 17, 300], 4, 2, d, causal, seed=d + causal, oracle_seqs=(0, 3, 7))


@pytest.mark.parametrize("causal", [True, False])
def test_mixed_lengths_single_heads(plx, causal):
    """Odd group size: a unit is two 64-row tiles of one head."""
    check(plx, [130, 5, 128, 257, 64], 3, 1, 128, causal, seed=5, oracle_seqs=(0, 1, 3))


def test_rho_none_and_one_sequence(plx):
    check(plx, [333], 4, 2, 128, True, seed=6, use_r=False, oracle_seqs=(0,))


def test_pretraining_width_mixed_batch(plx):
    """Hq=16, Hkv=8, d=128 with lengths from 1 to 4096 (16 sequences)."""
    lens = [4096, 1, 2048, 777, 1024, 3000, 64, 65, 512, 1500, 4000, 129, 333, 2500, 100, 900]
    check(plx, lens, 16, 8, 128, True, seed=7, oracle_seqs=(1, 6))
