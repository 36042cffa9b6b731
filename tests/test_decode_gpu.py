"""Decode (split-KV, balanced over the key tiles of the batch) on the GPU
against the fp64 oracle, through the C ABI."""
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


def run(plx, B, Hq, Hkv, S, d, seqlens="equal", seed=0, use_r=True, splits=0, r_scale=0.1, batches=None):
    q, kc, vc, r, sl = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=seed, seqlens=seqlens, r_scale=r_scale)
    dev = "cuda"
    out, lse = plx.plx_decode(q.to(dev), kc.to(dev), vc.to(dev), sl.to(dev), r.to(dev) if use_r else None,
                              num_splits=splits)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    ro, rl = oracle.decode_effective(q, r if use_r else None, kc, vc, sl, batches=batches)
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    if batches is not None:
        o, l, ro, rl = o[batches], l[batches], ro[batches], rl[batches]
    return o, l, ro, rl


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (16, 8), (8, 1), (24, 2)])
def test_decode_parity_shapes(plx, d, Hq, Hkv):
    o, l, ro, rl = run(plx, 3, Hq, Hkv, 200, d, seqlens=[200, 1, 130])
    assert_close(o, ro, l, rl, f"d={d} Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("S", [1, 2, 63, 64, 65, 127, 129, 1000])
def test_decode_ragged_lengths(plx, S):
    o, l, ro, rl = run(plx, 2, 4, 2, S, 128, seqlens=[S, max(1, S // 3)], seed=S)
    assert_close(o, ro, l, rl, f"S={S}")


def test_decode_empty_context(plx):
    q, kc, vc, r, sl = inputs.decode_inputs(3, 4, 2, 256, 128, seed=3, seqlens=[0, 256, -5])
    for splits in (1, 2, 0):
        out, lse = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), r.cuda(), num_splits=splits)
        o, l = out.float().cpu().numpy(), lse.cpu().numpy()
        assert (o[0] == 0).all() and (o[2] == 0).all()
        assert np.isneginf(l[0]).all() and np.isneginf(l[2]).all()
        ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
        assert_close(o, ro, l, rl, f"splits={splits}")


def test_decode_seqlen_clamped_to_cache(plx):
    q, kc, vc, r, _ = inputs.decode_inputs(2, 4, 2, 96, 64, seed=4)
    sl = torch.tensor([500, 96], dtype=torch.int32)
    out, lse = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), r.cuda())
    ro, rl = oracle.decode_effective(q, r, kc, vc, torch.tensor([96, 96]))
    assert_close(out, ro, lse, rl)


def test_decode_split_invariance(plx):
    q, kc, vc, r, sl = inputs.decode_inputs(4, 16, 8, 2048, 128, seed=5, seqlens="ragged")
    args = (q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), r.cuda())
    ref_o, ref_l = plx.plx_decode(*args, num_splits=1)
    ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
    assert_close(ref_o, ro, ref_l, rl, "splits=1")
    for s in (2, 3, 7, 16, 0):
        o, l = plx.plx_decode(*args, num_splits=s)
        assert_close(o, ro, l, rl, f"splits={s}")
        # different splits differ only by rounding
        assert (o.float() - ref_o.float()).abs().max().item() <= 1e-2


@pytest.mark.parametrize("splits", [1, 3, 5, 11, 0])
def test_decode_partitions_cross_sequences_and_head_groups(plx, splits):
    """The work partitions cut the tile list of the whole batch anywhere: in
    the middle of a sequence, of a head group (G = 12: groups of 8 and 4 query
    heads per KV head), next to empty sequences.  Every cut must merge back to
    the oracle's result."""
    lens = [0, 5, 0, 0, 300, 64, 0, 129, 1, 0]
    o, l, ro, rl = run(plx, len(lens), 24, 2, 320, 64, seqlens=lens, seed=40 + splits, splits=splits)
    assert_close(o, ro, l, rl, f"partitions={splits}")
    o, l, ro, rl = run(plx, len(lens), 24, 2, 320, 128, seqlens=lens, seed=50 + splits, splits=splits)
    assert_close(o, ro, l, rl, f"partitions={splits} d=128")


@pytest.mark.parametrize("B,S,d", [(40, 1000, 128), (300, 200, 128), (48, 700, 64), (700, 256, 64), (100, 128, 128),
                                   (160, 96, 64)])
def test_decode_many_segments(plx, B, S, d):
    """Batches with 128 (b, kv head) segments or more: of more than 256 keys
    they take the chunked plan (a CTA per chunk of a segment, chunk records
    merged per row), shorter ones the segment plan (one warp per whole
    segment, several segments per warp; 8 warps with 16-key stages for more
    than 4 x SMs segments of at most 128 keys); ragged lengths with empty
    sequences among them; sampled batch entries."""
    q, kc, vc, r, _ = inputs.decode_inputs(B, 16, 8, S, d, seed=60 + B, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(61)
    sl = torch.randint(0, S + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
    sl[::7] = 0
    sl[1] = S
    out, lse = plx.plx_decode(q, kc, vc, sl, r)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    n_ctas = plx.plx_decode_num_splits(B, 16, 8, S, d)
    assert (n_ctas >= B * 8) == (S > 256)  # chunked: a CTA per chunk of every segment
    if S <= 256:
        assert n_ctas * 4 < B * 8  # segment plan: warps hold several segments each
    pick = sorted({0, 1, 2, 7, B // 2, B - 1})
    qc, kcc, vcc, rc, slc = (t[pick].cpu() for t in (q, kc, vc, r, sl))
    ro, rl = oracle.decode_effective(qc, rc, kcc, vcc, slc)
    assert_close(out[pick], ro, lse[pick], rl, f"many segments B={B} S={S} d={d}")
    # the balanced plan (explicit partition count) gives the same result up to
    # rounding: its fp32 sums run in another order, so a bf16 output may land
    # one bf16 step (2^-8 relative, at most 2^-7 of the magnitude) away
    o2, l2 = plx.plx_decode(q, kc, vc, sl, r, num_splits=296)
    step = out.float().abs().clamp_min(1.0) * 2.0 ** -7
    assert bool(((o2.float() - out.float()).abs() <= step).all())


def test_decode_r_none_equals_r_zero_and_softmax(plx):
    q, kc, vc, r, sl = inputs.decode_inputs(2, 8, 4, 300, 128, seed=6, seqlens=[300, 123])
    a = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), None)
    b = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), torch.zeros_like(r).cuda())
    assert torch.equal(a[0], b[0])
    assert torch.allclose(a[1], b[1], rtol=0, atol=0)
    # rho = 0 is softmax attention: compare with torch SDPA in fp64 on the host
    qq = q.double()[:, :, None]
    for bb, n in enumerate([300, 123]):
        kk = kc.double()[bb:bb + 1, :, :n].repeat_interleave(2, 1)
        vv = vc.double()[bb:bb + 1, :, :n].repeat_interleave(2, 1)
        ref = torch.nn.functional.scaled_dot_product_attention(qq[bb:bb + 1], kk, vv)[0, :, 0]
        assert (a[0][bb].double().cpu() - ref).abs().max().item() < 1e-2


def test_decode_stress_inputs(plx):
    """Peaked scores, correlated values (large covariance) and a large probe."""
    B, Hq, Hkv, S, d = 2, 4, 2, 512, 128
    q, kc, vc, r, sl = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=7, r_scale=1.0, seqlens=[512, 400])
    q = (q.float() * 4).bfloat16()
    g = torch.Generator().manual_seed(8)
    W = torch.randn(d, d, generator=g) / d ** 0.5
    vc = (kc.float() @ W + 0.1 * torch.randn(kc.shape, generator=g)).bfloat16()
    out, lse = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), r.cuda())
    ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
    assert_close(out, ro, lse, rl, "stress", scale_abs=True)


@pytest.mark.parametrize("B", [1, 16, 64])
def test_decode_qwen3_layer_full_size(plx, B):
    """B in {1, 16, 64}, context 4096, Hq=16, Hkv=8, d=128, equal seqlens; the
    same launch configuration (automatic split count) the benchmark times."""
    o, l, ro, rl = run(plx, B, 16, 8, 4096, 128, seqlens="equal", seed=0)
    assert_close(o, ro, l, rl, f"B={B}")


def test_decode_sweep_point_ragged(plx):
    """A decode-sweep point with ragged seqlens in [ctx/2, ctx], sampled batches."""
    B, ctx = 256, 1024
    q, kc, vc, r, sl = inputs.decode_inputs(B, 16, 8, ctx, 128, seed=9, seqlens="ragged", device="cuda")
    out, lse = plx.plx_decode(q, kc, vc, sl, r)
    pick = [0, 1, 77, 128, 255]
    qc, kcc, vcc, rc, slc = (t[pick].cpu() for t in (q, kc, vc, r, sl))
    ro, rl = oracle.decode_effective(qc, rc, kcc, vcc, slc)
    assert_close(out[pick], ro, lse[pick], rl, "sweep point")


def test_decode_timeout_path_reports_and_recovers(plx):
    """A bounded wait that nothing completes: the kernel records a timeout,
    returns, and the context stays usable."""
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert plx.plx_selftest_wait_timeout(2_000_000) == plx.PLX_OK  # ~1 ms
    assert plx.plx_check_device_status() == plx.PLX_ERR_DEVICE_TIMEOUT
    assert plx.plx_check_device_status() == plx.PLX_OK  # cleared
    o, l, ro, rl = run(plx, 2, 4, 2, 128, 128, seed=11)
    assert_close(o, ro, l, rl, "after timeout")


def test_decode_largest_sweep_point(plx):
    """The largest decode-sweep point kept under the 150 GB cap: B=1024,
    context 32768 (137 GB of bf16 KV), ragged seqlens in [ctx/2, ctx], in the
    automatic split configuration the sweep times; sampled batch entries
    (first, last, random) against the oracle."""
    B, ctx = 1024, 32768
    free, _ = torch.cuda.mem_get_info()
    need = 2 * B * 8 * ctx * 128 * 2
    if free < need + (8 << 30):
        pytest.skip(f"needs {need / 1e9:.0f} GB of free device memory, {free / 1e9:.0f} GB free")
    q, kc, vc, r, sl = inputs.decode_inputs(B, 16, 8, ctx, 128, seed=10, seqlens="ragged", device="cuda")
    out, lse = plx.plx_decode(q, kc, vc, sl, r)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    pick = [0, 1, 511, 777, 1023]
    qc, kcc, vcc, rc, slc = (t[pick].cpu() for t in (q, kc, vc, r, sl))
    ro, rl = oracle.decode_effective(qc, rc, kcc, vcc, slc)
    assert_close(out[pick], ro, lse[pick], rl, "largest sweep point")
    del q, kc, vc, r, sl
    torch.cuda.empty_cache()


def _poison_tail(cache, seqlens):
    """A copy of cache [B, Hkv, S_max, d] whose rows at or past seqlens[b]
    hold NaN, +Inf and -Inf in turn (what an uninitialised cache may hold)."""
    bad = cache.clone()
    vals = (float("nan"), float("inf"), float("-inf"))
    for b, s in enumerate(seqlens.tolist()):
        s = max(0, min(int(s), cache.shape[2]))
        for row in range(s, cache.shape[2]):
            bad[b, :, row] = vals[row % 3]
    return bad


@pytest.mark.parametrize("B,Hq,Hkv,S,d,splits", [
    (3, 4, 2, 200, 128, 0),      # balanced plan, tails inside 16-key parts
    (3, 4, 2, 200, 64, 3),       # explicit partitions
    (5, 8, 1, 130, 128, 1),      # one partition over every segment
    (40, 16, 8, 1000, 128, 0),   # chunked plan (320 segments of > 256 keys)
    (100, 16, 8, 128, 128, 0),   # segment plan, 8 warps per CTA and 16-key stages (800 segments)
])
def test_decode_ignores_cache_rows_past_the_sequence(plx, B, Hq, Hkv, S, d, splits):
    """Keys past the sequence take no part whatever their rows hold: NaN and
    Inf there change no bit of out or lse."""
    rng = np.random.default_rng(B * 1000 + S)
    lens = [S] + [int(x) for x in rng.integers(1, S, size=B - 1)]
    lens[-1] = 65 if S > 65 else lens[-1]  # one key into a new tile
    q, kc, vc, r, sl = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=S + d, seqlens=lens)
    dev = "cuda"
    out0, lse0 = plx.plx_decode(q.to(dev), kc.to(dev), vc.to(dev), sl.to(dev), r.to(dev), num_splits=splits)
    kb, vb = _poison_tail(kc, sl), _poison_tail(vc, sl)
    out1, lse1 = plx.plx_decode(q.to(dev), kb.to(dev), vb.to(dev), sl.to(dev), r.to(dev), num_splits=splits)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
    ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
    assert_close(out1.float().cpu().numpy(), ro, lse1.cpu().numpy(), rl, f"poisoned tail B={B} S={S} d={d}")


def test_decode_paged_ignores_page_rows_past_the_sequence(plx):
    """The same on a paged cache: the rows of a sequence's last page past its
    length hold NaN / Inf."""
    B, Hq, Hkv, mp, ps, d = 4, 8, 2, 5, 64, 128
    q, kp, vp, r, table, _ = inputs.paged_decode_inputs(B, Hq, Hkv, mp, ps, d, seed=41)
    sl = torch.tensor([mp * ps, 1, 100, 257], dtype=torch.int32)
    kc, vc = inputs.gather_pages(kp, table), inputs.gather_pages(vp, table)
    kb, vb = kp.clone(), vp.clone()
    vals = (float("nan"), float("inf"), float("-inf"))
    for b in range(B):
        for key in range(int(sl[b]), mp * ps):
            page = int(table[b, key // ps])
            kb[page, :, key % ps] = vals[key % 3]
            vb[page, :, key % ps] = vals[(key + 1) % 3]
    dev = "cuda"
    args = (table.to(dev), sl.to(dev), r.to(dev))
    out0, lse0 = plx.plx_decode_paged(q.to(dev), kp.to(dev), vp.to(dev), *args)
    out1, lse1 = plx.plx_decode_paged(q.to(dev), kb.to(dev), vb.to(dev), *args)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)
    ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
    assert_close(out1.float().cpu().numpy(), ro, lse1.cpu().numpy(), rl, "paged poisoned tail")


def test_decode_records_ignore_cache_rows_past_the_sequence(plx):
    """The context-parallel form (state records of a key slice) with the
    slice's rows past each sequence poisoned: records identical bit for bit."""
    B, Hq, Hkv, S, d, off = 3, 4, 2, 150, 128, 100
    lens = [off + S, off + 70, off + 1]
    q, kc, vc, r, _ = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=77)
    sl = torch.tensor(lens, dtype=torch.int32)
    kb, vb = _poison_tail(kc, sl - off), _poison_tail(vc, sl - off)
    dev = "cuda"
    rec0 = plx.plx_decode_partial(q.to(dev), kc.to(dev), vc.to(dev), sl.to(dev), r.to(dev), key_offset=off).clone()
    rec1 = plx.plx_decode_partial(q.to(dev), kb.to(dev), vb.to(dev), sl.to(dev), r.to(dev), key_offset=off).clone()
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    assert torch.isfinite(rec1).all()
    assert torch.equal(rec0, rec1)


def test_decode_dirty_workspace_and_graph_replay(plx):
    """A workspace full of garbage gives the right answer (nothing in it needs
    to start at zero), and a CUDA graph that replays the same call (the
    balanced plan's two kernels, the second a programmatic dependent) gives
    it again, bit for bit."""
    B, Hq, Hkv, S, d, splits = 3, 8, 2, 1000, 128, 11
    q, kc, vc, r, sl = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=90, seqlens=[1000, 333, 777])
    dev = "cuda"
    q, kc, vc, r, sl_d = q.to(dev), kc.to(dev), vc.to(dev), r.to(dev), sl.to(dev)
    need = plx.plx_decode_workspace_size(B, Hq, Hkv, S, d, splits)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    plx.plx_decode(q, kc, vc, sl_d, r, num_splits=splits, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    ro, rl = oracle.decode_effective(q.cpu(), r.cpu(), kc.cpu(), vc.cpu(), sl)
    assert_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, "dirty workspace")
    want_o, want_l = out.clone(), lse.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        plx.plx_decode(q, kc, vc, sl_d, r, num_splits=splits, out=out, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        plx.plx_decode(q, kc, vc, sl_d, r, num_splits=splits, out=out, lse=lse, workspace=ws)
    for _ in range(3):
        out.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want_o) and torch.equal(lse, want_l)
    assert plx.plx_check_device_status() == plx.PLX_OK
    del g


@pytest.mark.parametrize("S,lens", [(256, [256, 255, 224, 33, 32, 31, 17, 16, 1, 0]), (64, [64, 63, 1, 0, 40, 64, 2, 9, 33, 32])])
@pytest.mark.parametrize("d,Hq,Hkv", [(128, 16, 8), (64, 24, 2), (128, 8, 8)])
def test_decode_segment_plan_lengths(plx, S, lens, d, Hq, Hkv):
    """The segment plan at every tail shape of its 32-key stages (a full
    stage, 1-31 keys in a last stage loaded in 16-key parts, empty
    sequences), GQA groups of more than 8 heads (two head groups per KV
    head), every row against the oracle."""
    B = len(lens)
    q, kc, vc, r, sl = inputs.decode_inputs(B, Hq, Hkv, S, d, seed=S + d + Hq, seqlens=lens)
    assert plx.plx_decode_workspace_size(B, Hq, Hkv, S, d, 0) >= 0
    out, lse = plx.plx_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), r.cuda())
    torch.cuda.synchronize()
    assert plx.plx_check_device_status() == plx.PLX_OK
    ro, rl = oracle.decode_effective(q, r, kc, vc, sl)
    assert_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, f"segment plan S={S} d={d} Hq={Hq}")
