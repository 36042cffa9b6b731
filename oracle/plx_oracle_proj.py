"""Plain fp64 CPU oracle for the projection in front of the Parallax attention.

THIS IS TEST INFRASTRUCTURE, under the same rule as ``plx_oracle``: only the
tests, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may use
it, and it shares nothing with the library.

What it computes.  The pages make the probe rho one more learned projection
of the layer input, next to the query, key and value projections
(news.chathome.org, "Parallax: a parameterized local linear attention ...",
section "What is Parallax"; gist.science, "Technical overview: Parallax ...",
"Method: Parallax / Core mechanism": rho_i is parameterised).  With the four
weight matrices stacked along the output dimension,

    W = [W_Q; W_K; W_V; W_R]     [Nout, d_model], one row per output feature,

the projection of token rows x [M, d_model] is y = x W^T, and its columns
are, in order, Hq heads of q, Hkv heads of k, Hkv heads of v and Hq heads of
rho, d columns per head.  Readings (the pages give no layout): the stacking
order q, k, v, rho; head-major columns within each block; token m of the
prefill input is position t = m mod N of sequence b = m div N.

Decode: one new token per sequence.  Its k and v are written into the cache
at row seqlens[b] of every KV head (the cache grows by one token per step;
zubnet.ai's Parallax page: a KV cache is still needed), and the sequence
length advances by one where the row exists.
"""
from __future__ import annotations

import numpy as np

__all__ = ["qkvr_projection", "qkvr_projection_decode"]


def _f64(t):
    if hasattr(t, "detach"):
        t = t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def _split_heads(y, B, N, H, d):
    """Columns [M, H*d] of one block -> [B, H, N, d]."""
    return y.reshape(B, N, H, d).transpose(0, 2, 1, 3)


def qkvr_projection(x, w, B, N, Hq, Hkv, d, with_r=True):
    """(q [B, Hq, N, d], k [B, Hkv, N, d], v, r [B, Hq, N, d] or None) from
    x [B*N, d_model] and w = [W_Q; W_K; W_V(; W_R)]."""
    x, w = _f64(x), _f64(w)
    nq, nkv = Hq * d, Hkv * d
    assert x.shape[0] == B * N and w.shape == (2 * nkv + (2 if with_r else 1) * nq, x.shape[1])
    y = x @ w.T
    q = _split_heads(y[:, :nq], B, N, Hq, d)
    k = _split_heads(y[:, nq:nq + nkv], B, N, Hkv, d)
    v = _split_heads(y[:, nq + nkv:nq + 2 * nkv], B, N, Hkv, d)
    r = _split_heads(y[:, nq + 2 * nkv:], B, N, Hq, d) if with_r else None
    return q, k, v, r


def qkvr_projection_decode(x, w, kcache, vcache, seqlens, Hq, with_r=True):
    """One decode step: x [B, d_model].  Returns (q [B, Hq, d], r or None,
    kcache', vcache' (copies with the new rows written), seqlens') where row
    seqlens[b] of every KV head of sequence b holds the token's k, v when
    0 <= seqlens[b] < S_max, and seqlens'[b] = seqlens[b] + 1 there."""
    kc, vc = _f64(kcache).copy(), _f64(vcache).copy()
    B, Hkv, S_max, d = kc.shape
    q, k, v, r = qkvr_projection(x, w, B, 1, Hq, Hkv, d, with_r)
    sl = np.asarray(_f64(seqlens), dtype=np.int64)
    out_sl = sl.copy()
    for b in range(B):
        s = int(sl[b])
        if 0 <= s < S_max:
            kc[b, :, s] = k[b, :, 0]
            vc[b, :, s] = v[b, :, 0]
            out_sl[b] = s + 1
    return q[:, :, 0], (r[:, :, 0] if with_r else None), kc, vc, out_sl
