"""The partial-state records of plx_fwd_partial and plx_decode_partial against
the oracle's streamed form (news.chathome.org, "Parallax: ...", section
"Hardware argument").

A record (m, l, c, pad, O1, O2) is unique only up to its reference maximum m
(any common rescaling of l, c, O1, O2 describes the same state), so each
record is compared through the quantities that do not depend on it: O1/l,
O2/l, c/l and the lse m + log2 l (m in log2 units on the device)."""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, MAX_ABS, REL_L2
from parameterized_local_linear_plx_b200 import inputs

pytestmark = pytest.mark.gpu

LN2 = 0.6931471805599453


@pytest.fixture(scope="module")
def plx():
    from parameterized_local_linear_plx_b200 import build
    build.build()
    from parameterized_local_linear_plx_b200 import plx as m
    assert torch.cuda.is_available()
    return m


def normalised_device(rec, d):
    """(O1/l, O2/l, c/l, lse) of device records [..., 2d + 4] (m in log2 units)."""
    rec = rec.double().cpu().numpy()
    m, l, c = rec[..., 0], rec[..., 1], rec[..., 2]
    return rec[..., 4:4 + d] / l[..., None], rec[..., 4 + d:4 + 2 * d] / l[..., None], c / l, (m + np.log2(l)) * LN2


def normalised_oracle(st):
    m, l, c, O1, O2 = st
    return O1 / l, O2 / l, c / l, m + np.log(l)


def compare(dev, ref, what):
    """The parity tolerances of every forward test, per quantity: max abs and
    relative L2 over the compared rows for O1/l, O2/l and c/l, abs for lse."""
    for got, want, name in zip(dev[:3], ref[:3], ("O1/l", "O2/l", "c/l")):
        err = np.abs(got - want).max()
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert err <= MAX_ABS, f"{what}: {name} max abs {err:.3e}"
        assert rel <= REL_L2, f"{what}: {name} rel L2 {rel:.3e}"
    assert np.abs(dev[3] - ref[3]).max() <= LSE_ABS, f"{what}: lse"


def f64(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_records(plx, causal, d):
    B, Hq, Hkv, N = 1, 4, 2, 200
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=21 + d, device="cuda")
    rec = plx.plx_fwd_partial(q, k, v, r, causal=causal)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    dev = normalised_device(rec, d)
    qn, kn, vn, rn = f64(q), f64(k), f64(v), f64(r)
    scale = 1.0 / np.sqrt(d)
    G = Hq // Hkv
    for h in range(Hq):
        ref = [np.empty((N, d)), np.empty((N, d)), np.empty(N), np.empty(N)]
        for i in range(N):
            n = i + 1 if causal else N
            st = oracle.chunk_state(qn[0, h, i], rn[0, h, i], kn[0, h // G, :n], vn[0, h // G, :n], scale)
            for x, y in zip(ref, normalised_oracle(st)):
                x[i] = y
        compare(tuple(x[0, h] for x in dev), tuple(ref), f"prefill record h={h} causal={causal} d={d}")


def test_decode_records(plx):
    B, Hq, Hkv, S, d = 3, 4, 2, 300, 128
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=33, device="cuda")
    sl = torch.tensor([1, 150, 300], dtype=torch.int32, device="cuda")
    rec = plx.plx_decode_partial(q, kc, vc, sl, r, num_splits=3)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    dev = normalised_device(rec, d)
    qn, kn, vn, rn = f64(q), f64(kc), f64(vc), f64(r)
    scale = 1.0 / np.sqrt(d)
    G = Hq // Hkv
    # one record per (b, h): compared over all B * Hq rows at once, as every
    # parity test compares over the whole tensor (c/l of a single row is one
    # scalar, whose relative error alone says nothing when it is near zero)
    ref = [np.empty((B, Hq, d)), np.empty((B, Hq, d)), np.empty((B, Hq)), np.empty((B, Hq))]
    for b in range(B):
        n = int(sl[b])
        for h in range(Hq):
            st = oracle.chunk_state(qn[b, h], rn[b, h], kn[b, h // G, :n], vn[b, h // G, :n], scale)
            for x, y in zip(ref, normalised_oracle(st)):
                x[b, h] = y
    compare(dev, tuple(ref), "decode records")
