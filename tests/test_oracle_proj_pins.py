"""Pins of the projection oracle (oracle/plx_oracle_proj.py) against values
worked by hand (tests/golden/proj_hand_examples.json), against a library
linear map, and against planted mistakes in its layout (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import plx_oracle_proj as op

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "proj_hand_examples.json")


def load():
    with open(GOLDEN) as f:
        return json.load(f)


def stack(ex, with_r=True):
    blocks = [ex["W_Q"], ex["W_K"], ex["W_V"]] + ([ex["W_R"]] if with_r else [])
    return np.concatenate([np.asarray(b, dtype=np.float64) for b in blocks])


@pytest.mark.parametrize("i", [0, 1])
def test_prefill_hand_examples(i):
    ex = load()["prefill"][i]
    q, k, v, r = op.qkvr_projection(np.asarray(ex["x"], float), stack(ex), ex["B"], ex["N"], ex["Hq"], ex["Hkv"],
                                    ex["d"])
    for got, name in ((q, "q"), (k, "k"), (v, "v"), (r, "r")):
        assert np.array_equal(got, np.asarray(ex[name], float)), name
    q2, k2, v2, r2 = op.qkvr_projection(np.asarray(ex["x"], float), stack(ex, False), ex["B"], ex["N"], ex["Hq"],
                                        ex["Hkv"], ex["d"], with_r=False)
    assert r2 is None and np.array_equal(q2, q) and np.array_equal(k2, k) and np.array_equal(v2, v)


def test_decode_hand_example():
    ex = load()["decode"][0]
    x = np.asarray(ex["x"], float)
    B = x.shape[0]
    kc = np.full((B, 1, ex["S_max"], 1), float(ex["cache_fill"]))
    vc = kc.copy()
    q, r, kc2, vc2, sl = op.qkvr_projection_decode(x, stack(ex), kc, vc, np.asarray(ex["seqlens"]), ex["Hq"])
    assert np.array_equal(q, np.asarray(ex["q"], float).reshape(q.shape))
    assert np.array_equal(r, np.asarray(ex["r"], float).reshape(r.shape))
    assert np.array_equal(kc2, np.asarray(ex["kcache"], float))
    assert np.array_equal(vc2, np.asarray(ex["vcache"], float))
    assert list(sl) == ex["seqlens_out"]
    assert (kc == ex["cache_fill"]).all()  # the inputs are not modified


def test_matches_a_library_linear_map():
    g = torch.Generator().manual_seed(0)
    B, N, dm, Hq, Hkv, d = 2, 5, 24, 4, 2, 8
    x = torch.randn(B * N, dm, generator=g, dtype=torch.float64)
    w = torch.randn((2 * Hq + 2 * Hkv) * d, dm, generator=g, dtype=torch.float64)
    y = torch.nn.functional.linear(x, w).numpy()
    q, k, v, r = op.qkvr_projection(x, w, B, N, Hq, Hkv, d)
    for b in range(B):
        for t in range(N):
            m = b * N + t
            for h in range(Hq):
                assert np.allclose(q[b, h, t], y[m, h * d:(h + 1) * d], atol=1e-12)
                off = (Hq + 2 * Hkv) * d
                assert np.allclose(r[b, h, t], y[m, off + h * d:off + (h + 1) * d], atol=1e-12)
            for h in range(Hkv):
                assert np.allclose(k[b, h, t], y[m, Hq * d + h * d:Hq * d + (h + 1) * d], atol=1e-12)
                off = (Hq + Hkv) * d
                assert np.allclose(v[b, h, t], y[m, off + h * d:off + (h + 1) * d], atol=1e-12)


def test_planted_layout_mistakes_are_caught():
    """Copies of the oracle with a plausible mistake each disagree with the
    hand-worked layout example."""
    ex = load()["prefill"][1]
    x, w = np.asarray(ex["x"], float), stack(ex)
    B, N, Hq, Hkv, d = ex["B"], ex["N"], ex["Hq"], ex["Hkv"], ex["d"]
    want_q, want_k = np.asarray(ex["q"], float), np.asarray(ex["k"], float)

    def token_major_heads(y, H):  # heads and tokens swapped
        return y.reshape(B, H, N, d)

    def swapped_kv(xx, ww):
        nq, nkv = Hq * d, Hkv * d
        ww = np.concatenate([ww[:nq], ww[nq + nkv:nq + 2 * nkv], ww[nq:nq + nkv], ww[nq + 2 * nkv:]])
        return op.qkvr_projection(xx, ww, B, N, Hq, Hkv, d)

    y = x @ w.T
    assert np.array_equal(op.qkvr_projection(x, w, B, N, Hq, Hkv, d)[0], want_q)
    assert not np.array_equal(token_major_heads(y[:, :Hq * d], Hq), want_q)
    assert not np.array_equal(swapped_kv(x, w)[1], want_k)
    # token m read as t * B + b instead of b * N + t
    assert not np.array_equal(y[:, :Hq * d].reshape(N, B, Hq, d).transpose(1, 2, 0, 3), want_q)
