"""The C ABI without a GPU: the library loads, exports every entry point that
include/plx.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "plx.h")


@pytest.fixture(scope="module")
def plx():
    from parameterized_local_linear_plx_b200 import build
    build.build()
    from parameterized_local_linear_plx_b200 import plx as m
    return m


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(plx_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ["plx_fwd", "plx_fwd_train", "plx_bwd", "plx_bwd_workspace_size", "plx_decode_paged", "plx_kv_append", "plx_kv_append_paged", "plx_fwd_varlen", "plx_decode_partial", "plx_decode_merge", "plx_decode_partial_size",
              "plx_fwd_partial", "plx_fwd_partial_size", "plx_fwd_merge",
              "plx_decode", "plx_decode_workspace_size", "plx_decode_num_splits",
              "plx_check_device_status", "plx_status_string", "plx_version", "plx_selftest_wait_timeout"]:
        assert n in names


def test_library_exports_every_declared_symbol(plx):
    out = subprocess.run(["nm", "-D", "--defined-only", plx.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (plx_[a-z0-9_]+)\b", out))
    missing = [n for n in declared_entry_points() if n not in exported]
    assert not missing, missing
    for n in declared_entry_points():
        assert hasattr(plx.lib, n)


def test_header_is_plain_c():
    """The header compiles as C99 with no CUDA or torch includes."""
    src = '#include "plx.h"\nint main(void){ return plx_version() > 0 ? 0 : 1; }\n'
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.dirname(HEADER),
                          "-x", "c", "-"], input=src, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_status_strings(plx):
    for code in range(-9, 1):
        s = plx.plx_status_string(code)
        assert s.startswith("PLX_")
    assert "unknown" in plx.plx_status_string(-100)
    assert plx.plx_version() >= 100


P = ctypes.c_void_p
A = 0x10000  # a 16-byte aligned fake device address; never dereferenced on these paths


def fwd(plx, q=A, k=A, v=A, r=A, out=A, lse=A, B=1, Hq=2, Hkv=1, N=8, d=64, causal=1):
    return plx.lib.plx_fwd(P(q), P(k), P(v), P(r), P(out), P(lse), B, Hq, Hkv, N, d, causal, 0.125, None)


def dec(plx, q=A, r=A, kc=A, vc=A, sl=A, out=A, lse=A, B=1, Hq=2, Hkv=1, S=64, d=64, splits=1, ws=None, wsb=0):
    return plx.lib.plx_decode(P(q), P(r), P(kc), P(vc), P(sl), P(out), P(lse), B, Hq, Hkv, S, d, 0.125,
                              splits, P(ws), wsb, None)


def test_fwd_argument_errors(plx):
    assert fwd(plx, q=None) == plx.PLX_ERR_NULL
    assert fwd(plx, k=None) == plx.PLX_ERR_NULL
    assert fwd(plx, v=None) == plx.PLX_ERR_NULL
    assert fwd(plx, out=None) == plx.PLX_ERR_NULL
    for kw in [dict(B=0), dict(Hq=0), dict(Hkv=0), dict(N=0), dict(N=-3)]:
        assert fwd(plx, **kw) == plx.PLX_ERR_SHAPE, kw
    for d in [0, 32, 96, 256]:
        assert fwd(plx, d=d) == plx.PLX_ERR_HEADDIM
    assert fwd(plx, Hq=3, Hkv=2) == plx.PLX_ERR_GQA
    assert fwd(plx, q=A + 8) == plx.PLX_ERR_ALIGN
    assert fwd(plx, r=A + 2) == plx.PLX_ERR_ALIGN
    assert fwd(plx, lse=A + 2) == plx.PLX_ERR_ALIGN


def test_decode_argument_errors(plx):
    assert dec(plx, q=None) == plx.PLX_ERR_NULL
    assert dec(plx, kc=None) == plx.PLX_ERR_NULL
    assert dec(plx, sl=None) == plx.PLX_ERR_NULL
    assert dec(plx, B=0) == plx.PLX_ERR_SHAPE
    assert dec(plx, S=0) == plx.PLX_ERR_SHAPE
    assert dec(plx, splits=-1) == plx.PLX_ERR_SHAPE
    assert dec(plx, d=100) == plx.PLX_ERR_HEADDIM
    assert dec(plx, Hq=5, Hkv=2) == plx.PLX_ERR_GQA
    assert dec(plx, vc=A + 4) == plx.PLX_ERR_ALIGN
    assert dec(plx, sl=A + 2) == plx.PLX_ERR_ALIGN
    # every call needs the workspace (partial states of the partitions)
    assert dec(plx, S=256, splits=2) == plx.PLX_ERR_WORKSPACE
    need = plx.plx_decode_workspace_size(1, 2, 1, 256, 64, 2)
    assert dec(plx, S=256, splits=2, ws=A, wsb=need - 1) == plx.PLX_ERR_WORKSPACE
    assert dec(plx, S=256, splits=2, ws=A + 4, wsb=need) == plx.PLX_ERR_ALIGN


def test_split_planning(plx):
    # P partitions (persistent CTAs): two partial slots of min(G, 8) rows of
    # (2d + 4) floats per partition, padded to 256 bytes; B and S_max do not enter
    up = lambda n: (n + 255) // 256 * 256
    for (Hq, Hkv, d, P) in [(4, 2, 128, 4), (16, 8, 128, 296), (8, 2, 64, 7), (16, 1, 128, 3)]:
        want = up(2 * P * min(Hq // Hkv, 8) * (2 * d + 4) * 4)
        assert plx.plx_decode_workspace_size(2, Hq, Hkv, 1024, d, P) == want
        assert plx.plx_decode_workspace_size(64, Hq, Hkv, 32768, d, P) == want
    # automatic plan, few segments (b, kv head): one balanced partition per SM
    n = plx.plx_decode_num_splits(1, 16, 8, 4096, 128)
    assert n >= 1
    assert plx.plx_decode_num_splits(8, 16, 8, 32768, 128) == n  # 64 segments
    assert plx.plx_decode_workspace_size(1, 16, 8, 4096, 128, 0) == plx.plx_decode_workspace_size(1, 16, 8, 4096, 128, n)
    # automatic plan, many segments: chunks of whole 64-key tiles, about four
    # waves of two CTAs per SM, chunks of at least 128 keys; one record of
    # (2d + 4) floats per (b, h, chunk) when a segment has several chunks
    sms = n
    for B, S in [(64, 4096), (256, 1024), (2048, 16384), (1024, 512)]:
        segs = B * 8
        sp = max(1, min(-(-4 * 2 * sms // segs), (S + 127) // 128))
        tiles = -(-(-(-S // sp)) // 64)
        splits = -(-S // (tiles * 64))
        assert plx.plx_decode_num_splits(B, 16, 8, S, 128) == segs * splits
        assert plx.plx_decode_workspace_size(B, 16, 8, S, 128, 0) == (up(B * 16 * splits * 260 * 4) if splits > 1 else 0)
    assert plx.plx_decode_num_splits(2048, 16, 8, 16384, 128) == 2048 * 8  # one chunk per segment: no workspace
    # short segments (at most 256 keys): the segment plan, one warp per whole
    # segment, segments dealt round the CTAs first, at most one CTA per SM and
    # no more CTAs than segments, no workspace of its own; the workspace size
    # covers the paged call, which keeps the balanced plan (two partitions
    # per SM for short segments)
    assert plx.plx_decode_num_splits(2048, 16, 8, 256, 128) == n
    assert plx.plx_decode_num_splits(1, 16, 8, 128, 128) == 8  # 8 segments: 8 CTAs
    assert plx.plx_decode_workspace_size(1, 16, 8, 128, 128, 0) == up(2 * (2 * n) * 2 * 260 * 4)
    # bad shapes: size 0
    assert plx.plx_decode_workspace_size(1, 3, 2, 128, 128, 2) == 0
    assert plx.plx_decode_workspace_size(1, 2, 1, 128, 128, -1) == 0


def fwdt(plx, q=A, k=A, v=A, r=A, out=A, lse=A, obar=A, sbar=A, B=1, Hq=2, Hkv=1, N=8, d=64):
    return plx.lib.plx_fwd_train(P(q), P(k), P(v), P(r), P(out), P(lse), P(obar), P(sbar), B, Hq, Hkv, N, d, 1,
                                 0.125, None)


def bwd(plx, ws=A, wsb=None, B=1, Hq=2, Hkv=1, N=8, d=64, **ptrs):
    names = ["q", "k", "v", "r", "out", "dout", "lse", "obar", "sbar", "dq", "dk", "dv", "dr"]
    vals = [P(ptrs.get(n, A)) for n in names]
    if wsb is None:
        wsb = plx.plx_bwd_workspace_size(B, Hq, Hkv, N, d)
    return plx.lib.plx_bwd(*vals, B, Hq, Hkv, N, d, 1, 0.125, P(ws), wsb, None)


def test_train_forward_argument_errors(plx):
    assert fwdt(plx, lse=None) == plx.PLX_ERR_NULL
    assert fwdt(plx, obar=None) == plx.PLX_ERR_NULL
    assert fwdt(plx, sbar=None) == plx.PLX_ERR_NULL          # rho given: s_bar required
    assert fwdt(plx, q=None) == plx.PLX_ERR_NULL
    assert fwdt(plx, N=0) == plx.PLX_ERR_SHAPE
    assert fwdt(plx, d=80) == plx.PLX_ERR_HEADDIM
    assert fwdt(plx, obar=A + 8) == plx.PLX_ERR_ALIGN
    assert fwdt(plx, sbar=A + 1) == plx.PLX_ERR_ALIGN


def test_bwd_workspace_size(plx):
    # two fp32 arrays of B * Hq * N, each padded to 256 bytes
    assert plx.plx_bwd_workspace_size(2, 4, 2, 100, 128) == 2 * 3328
    assert plx.plx_bwd_workspace_size(1, 1, 1, 64, 64) == 2 * 256
    assert plx.plx_bwd_workspace_size(0, 4, 2, 100, 128) == 0
    assert plx.plx_bwd_workspace_size(1, 3, 2, 100, 128) == 0
    assert plx.plx_bwd_workspace_size(1, 4, 2, 100, 96) == 0


def test_bwd_argument_errors(plx):
    for n in ["q", "k", "v", "out", "dout", "lse", "obar", "dq", "dk", "dv"]:
        assert bwd(plx, **{n: None}) == plx.PLX_ERR_NULL, n
    assert bwd(plx, sbar=None) == plx.PLX_ERR_NULL           # rho given: s_bar required
    assert bwd(plx, N=0) == plx.PLX_ERR_SHAPE
    assert bwd(plx, d=32) == plx.PLX_ERR_HEADDIM
    assert bwd(plx, Hq=3, Hkv=2) == plx.PLX_ERR_GQA
    assert bwd(plx, dk=A + 8) == plx.PLX_ERR_ALIGN
    assert bwd(plx, dr=A + 8) == plx.PLX_ERR_ALIGN
    assert bwd(plx, lse=A + 2) == plx.PLX_ERR_ALIGN
    assert bwd(plx, ws=None) == plx.PLX_ERR_WORKSPACE
    assert bwd(plx, wsb=plx.plx_bwd_workspace_size(1, 2, 1, 8, 64) - 1) == plx.PLX_ERR_WORKSPACE


def paged(plx, q=A, r=A, kp=A, vp=A, bt=A, sl=A, out=A, lse=A, B=1, Hq=2, Hkv=1, num_pages=4, ps=16, mp=2,
          d=64, splits=1, ws=None, wsb=0):
    return plx.lib.plx_decode_paged(P(q), P(r), P(kp), P(vp), P(bt), P(sl), P(out), P(lse), B, Hq, Hkv, num_pages,
                                    ps, mp, d, 0.125, splits, P(ws), wsb, None)


def test_paged_decode_argument_errors(plx):
    for kw in [dict(q=None), dict(kp=None), dict(vp=None), dict(bt=None), dict(sl=None), dict(out=None)]:
        assert paged(plx, **kw) == plx.PLX_ERR_NULL, kw
    for ps in [0, 8, 24, 100, 8192]:
        assert paged(plx, ps=ps) == plx.PLX_ERR_SHAPE, ps
    for kw in [dict(B=0), dict(num_pages=0), dict(mp=0), dict(splits=-1)]:
        assert paged(plx, **kw) == plx.PLX_ERR_SHAPE, kw
    assert paged(plx, d=96) == plx.PLX_ERR_HEADDIM
    assert paged(plx, Hq=3, Hkv=2) == plx.PLX_ERR_GQA
    assert paged(plx, kp=A + 8) == plx.PLX_ERR_ALIGN
    assert paged(plx, bt=A + 2) == plx.PLX_ERR_ALIGN
    need = plx.plx_decode_workspace_size(1, 2, 1, 16 * 32, 64, 2)
    assert paged(plx, mp=32, splits=2) == plx.PLX_ERR_WORKSPACE
    assert paged(plx, mp=32, splits=2, ws=A, wsb=need - 1) == plx.PLX_ERR_WORKSPACE


def test_kv_append_argument_errors(plx):
    ap = plx.lib.plx_kv_append
    assert ap(P(None), P(A), P(A), P(A), P(A), 1, 1, 8, 64, 1, None) == plx.PLX_ERR_NULL
    assert ap(P(A), P(A), P(A), P(A), P(None), 1, 1, 8, 64, 1, None) == plx.PLX_ERR_NULL
    assert ap(P(A), P(A), P(A), P(A), P(A), 0, 1, 8, 64, 1, None) == plx.PLX_ERR_SHAPE
    assert ap(P(A), P(A), P(A), P(A), P(A), 1, 1, 0, 64, 1, None) == plx.PLX_ERR_SHAPE
    assert ap(P(A), P(A), P(A), P(A), P(A), 1, 1, 8, 80, 1, None) == plx.PLX_ERR_HEADDIM
    assert ap(P(A + 8), P(A), P(A), P(A), P(A), 1, 1, 8, 64, 1, None) == plx.PLX_ERR_ALIGN
    apg = plx.lib.plx_kv_append_paged
    assert apg(P(A), P(A), P(A), P(A), P(None), P(A), 1, 1, 4, 16, 2, 64, 1, None) == plx.PLX_ERR_NULL
    assert apg(P(A), P(A), P(A), P(A), P(A), P(A), 1, 1, 4, 24, 2, 64, 1, None) == plx.PLX_ERR_SHAPE
    assert apg(P(A), P(A), P(A), P(A), P(A), P(A), 1, 1, 0, 16, 2, 64, 1, None) == plx.PLX_ERR_SHAPE
    assert apg(P(A), P(A), P(A), P(A), P(A + 2), P(A), 1, 1, 4, 16, 2, 64, 1, None) == plx.PLX_ERR_ALIGN


def test_varlen_argument_errors(plx):
    vf = plx.lib.plx_fwd_varlen
    args = lambda **kw: [P(kw.get(n, A)) for n in ("q", "k", "v", "r", "out", "lse", "cu")]
    assert vf(*args(cu=None), 2, 2, 1, 100, 64, 64, 1, 0.125, None) == plx.PLX_ERR_NULL
    assert vf(*args(q=None), 2, 2, 1, 100, 64, 64, 1, 0.125, None) == plx.PLX_ERR_NULL
    assert vf(*args(), 2, 2, 1, 0, 64, 64, 1, 0.125, None) == plx.PLX_ERR_SHAPE      # total < 1
    assert vf(*args(), 2, 2, 1, 100, 0, 64, 1, 0.125, None) == plx.PLX_ERR_SHAPE     # max_seqlen < 1
    assert vf(*args(), 2, 2, 1, 100, 64, 48, 1, 0.125, None) == plx.PLX_ERR_HEADDIM
    assert vf(*args(), 2, 3, 2, 100, 64, 64, 1, 0.125, None) == plx.PLX_ERR_GQA
    assert vf(*args(cu=A + 2), 2, 2, 1, 100, 64, 64, 1, 0.125, None) == plx.PLX_ERR_ALIGN


def test_partial_and_merge_argument_errors(plx):
    dp = plx.lib.plx_decode_partial
    ok = lambda **kw: [P(kw.get(n, A)) for n in ("q", "r", "kc", "vc", "sl")]
    need = plx.plx_decode_partial_size(1, 2, 1, 64, 64, 1)
    # the records [B, Hq, 2d + 4] fp32, then the workspace of one partition
    up = lambda n: (n + 255) // 256 * 256
    assert need == up(1 * 2 * (2 * 64 + 4) * 4) + plx.plx_decode_workspace_size(1, 2, 1, 64, 64, 1)
    assert dp(*ok(), 0, 1, 2, 1, 64, 64, 0.125, 1, P(None), need, None) == plx.PLX_ERR_NULL
    assert dp(*ok(), -1, 1, 2, 1, 64, 64, 0.125, 1, P(A), need, None) == plx.PLX_ERR_SHAPE
    assert dp(*ok(), 0, 1, 2, 1, 64, 64, 0.125, 1, P(A), need - 4, None) == plx.PLX_ERR_WORKSPACE
    assert dp(*ok(kc=None), 0, 1, 2, 1, 64, 64, 0.125, 1, P(A), need, None) == plx.PLX_ERR_NULL
    assert dp(*ok(), 0, 1, 2, 1, 64, 96, 0.125, 1, P(A), need, None) == plx.PLX_ERR_HEADDIM
    mg = plx.lib.plx_decode_merge
    assert mg(P(None), 2, 1, 2, 64, P(A), P(A), None) == plx.PLX_ERR_NULL
    assert mg(P(A), 0, 1, 2, 64, P(A), P(A), None) == plx.PLX_ERR_SHAPE
    assert mg(P(A), 2, 0, 2, 64, P(A), P(A), None) == plx.PLX_ERR_SHAPE
    assert mg(P(A), 2, 1, 2, 80, P(A), P(A), None) == plx.PLX_ERR_HEADDIM
    assert mg(P(A + 4), 2, 1, 2, 64, P(A), P(A), None) == plx.PLX_ERR_ALIGN
    assert mg(P(A), 2, 1, 2, 64, P(A + 4), P(A), None) == plx.PLX_ERR_ALIGN


def test_prefill_partial_and_merge_argument_errors(plx):
    fp = plx.lib.plx_fwd_partial
    need = plx.plx_fwd_partial_size(1, 2, 64, 64)
    assert need == 1 * 2 * 64 * (2 * 64 + 4) * 4
    assert plx.plx_fwd_partial_size(1, 2, 64, 96) == 0 and plx.plx_fwd_partial_size(0, 2, 64, 64) == 0
    qkv = [P(A), P(A), P(A), P(None)]
    assert fp(*qkv, P(None), need, 1, 2, 1, 64, 64, 1, 0.125, None) == plx.PLX_ERR_NULL
    assert fp(*qkv, P(A), need - 4, 1, 2, 1, 64, 64, 1, 0.125, None) == plx.PLX_ERR_WORKSPACE
    assert fp(P(A), P(None), P(A), P(None), P(A), need, 1, 2, 1, 64, 64, 1, 0.125, None) == plx.PLX_ERR_NULL
    assert fp(*qkv, P(A), need, 1, 2, 1, 64, 96, 1, 0.125, None) == plx.PLX_ERR_HEADDIM
    assert fp(*qkv, P(A), 1 << 40, 1, 3, 2, 64, 64, 1, 0.125, None) == plx.PLX_ERR_GQA
    assert fp(*qkv, P(A + 4), need, 1, 2, 1, 64, 64, 1, 0.125, None) == plx.PLX_ERR_ALIGN
    assert fp(*qkv, P(A), need, 1, 2, 1, 0, 64, 1, 0.125, None) == plx.PLX_ERR_SHAPE
    mg = plx.lib.plx_fwd_merge
    assert mg(P(None), 2, 1, 2, 64, 64, P(A), P(A), None) == plx.PLX_ERR_NULL
    assert mg(P(A), 0, 1, 2, 64, 64, P(A), P(A), None) == plx.PLX_ERR_SHAPE
    assert mg(P(A), 2, 1, 2, 0, 64, P(A), P(A), None) == plx.PLX_ERR_SHAPE
    assert mg(P(A), 2, 1, 2, 64, 80, P(A), P(A), None) == plx.PLX_ERR_HEADDIM
    assert mg(P(A + 4), 2, 1, 2, 64, 64, P(A), P(A), None) == plx.PLX_ERR_ALIGN
