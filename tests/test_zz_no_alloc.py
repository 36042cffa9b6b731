"""plx_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a plugin that is handed only its input
and output buffers by the runtime that owns device memory, or a serving loop
that forbids device allocation after start-up).  plx_decode_noalloc keeps the
split partial states in the library's fixed device scratch array instead of
a caller workspace.  These tests call it through the C ABI (the raw ctypes
handle) and compare it with plx_decode, the entry point that takes a
workspace, within the parity tolerances used by every GPU test.  The file is
named so that pytest collects it last.
"""
import ctypes

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
    assert m.plx_check_device_status() == m.PLX_OK
    return m


def _noalloc(plx, q, kc, vc, sl, r, num_splits):
    """Call the C entry point directly; output buffers come from the caller."""
    B, Hq, d = q.shape
    Hkv, S_max = kc.shape[1], kc.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    P = ctypes.c_void_p
    st = plx.lib.plx_decode_noalloc(
        P(q.data_ptr()), P(r.data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()), P(sl.data_ptr()),
        P(out.data_ptr()), P(lse.data_ptr()), B, Hq, Hkv, S_max, d, d ** -0.5, num_splits,
        P(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def test_noalloc_matches_decode_on_two_calls_in_a_row(plx):
    # two different problems back to back: the shared scratch keeps the first
    # call's partials, and the second call must not depend on them
    cases = [dict(B=4, Hq=16, Hkv=8, S=2048, d=128, seed=31, seqlens="ragged", splits=4),
             dict(B=3, Hq=8, Hkv=2, S=1000, d=64, seed=32, seqlens=[1000, 17, 640], splits=0)]
    for c in cases:
        q, kc, vc, r, sl = inputs.decode_inputs(c["B"], c["Hq"], c["Hkv"], c["S"], c["d"], seed=c["seed"],
                                                seqlens=c["seqlens"], device="cuda")
        need = plx.plx_decode_workspace_size(c["B"], c["Hq"], c["Hkv"], c["S"], c["d"], c["splits"])
        assert 0 < need <= plx.PLX_NOALLOC_SCRATCH_BYTES  # the scratch array is really used
        ref_o, ref_l = plx.plx_decode(q, kc, vc, sl, r, num_splits=c["splits"])
        st, out, lse = _noalloc(plx, q, kc, vc, sl, r, c["splits"])
        assert st == plx.PLX_OK, plx.plx_status_string(st)
        torch.cuda.synchronize()
        assert plx.plx_check_device_status() == plx.PLX_OK
        assert_close(out, ref_o, lse, ref_l, f"noalloc vs decode {c}")
        or_o, or_l = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), sl.cpu())
        assert_close(out, or_o, lse, or_l, f"noalloc vs oracle {c}")


def test_noalloc_rejects_requests_above_its_scratch(plx):
    # 8192 work partitions: their partial-state slots would need ~34 MB > 16 MiB
    B, Hq, Hkv, S, d, splits = 64, 16, 8, 65536, 128, 8192
    need = plx.plx_decode_workspace_size(B, Hq, Hkv, S, d, splits)
    assert need > plx.PLX_NOALLOC_SCRATCH_BYTES
    P = ctypes.c_void_p
    A = P(0x10000)  # never dereferenced: the size check comes before any launch
    st = plx.lib.plx_decode_noalloc(A, A, A, A, A, A, A, B, Hq, Hkv, S, d, 0.1, splits, None)
    assert st == plx.PLX_ERR_WORKSPACE
