"""Plain fp64 CPU oracle for the Parallax attention forward pass.

THIS IS TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py`` may import it. The
library's product path never calls anything here, and nothing here calls the
library: the two share no code, no constants and no helpers.

What it computes, and where the pages say so
--------------------------------------------
Sources are cited by page and section:

[GIST]  gist.science, "Technical overview: Parallax - parameterized local
        linear attention for language modeling" (Japanese), section
        "Method: Parallax / Core mechanism": the output equation
        o^PLX_i = o^SA_i - Sigma^(i)_KV rho_i, with o^SA_i the standard softmax
        attention output and Sigma^(i)_KV the KV covariance matrix; and the
        bullet "removing boundary amplification": eta_i is set to zero.
[CHAT]  news.chathome.org, "Parallax: a parameterized local linear attention
        that keeps Softmax and adds a learned covariance correction branch"
        (Chinese), section "What is Parallax": softmax attention is the
        Nadaraya-Watson (local constant) estimator; section "How the
        mechanism works": output = softmax output minus the projected
        covariance term; the boundary factor is set to zero; probe norm zero
        reduces exactly to softmax attention.

The pages leave open some details; the readings taken here are:
  * Sigma^(i)_KV is the softmax-weighted (w_ij, normalised, no Bessel
    correction) covariance of values against keys, a d_v x d_k matrix, so
    Sigma rho is a value-space vector and rho lives in key space.
  * s_ij = rho_i . k_j is not scaled by 1/sqrt(d); only q.k is.
  * Causal prefill uses the keys j <= i (diagonal included); non-causal uses
    every key; decode uses the cached keys j < seqlen[b].
  * GQA: query head h reads key/value head floor(h / G), G = Hq / Hkv;
    rho is given per query head.
  * lse is the natural-log log-sum-exp of the scaled q.k scores (branch 1).
  * An empty key set (decode seqlen <= 0) gives o = 0 and lse = -inf.

Two independent forms are provided.

1. ``*_explicit``: the definition written out.  Per query row: softmax
   weights w, weighted means k_bar and o_bar, the explicit d x d matrix
   Sigma_KV = sum_j w_j (v_j - o_bar)(k_j - k_bar)^T, and o = o_bar - Sigma rho.
   Cost ~2 d^2 per key: for small inputs and sampled rows.

2. ``*_effective``: the same quantity rewritten with effective weights.
   Because sum_j w_j (k_j - k_bar) = 0,
       Sigma rho = sum_j w_j v_j (s_j - s_bar),   s_j = rho.k_j,  s_bar = sum_j w_j s_j,
   so o = sum_j w_j (1 - (s_j - s_bar)) v_j.  The effective weights sum to 1
   and can be negative or exceed 1 (news.chathome.org, section "Score
   differences").  Whole (b, head) blocks as matrices: for full tensors.

Neither form implements the streamed (online max / rescale) algorithm that
the kernels use.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "softmax_row",
    "parallax_row_explicit",
    "prefill_explicit",
    "prefill_rows_explicit",
    "prefill_effective",
    "decode_explicit",
    "decode_rows_explicit",
    "decode_effective",
]


def _f64(x):
    """Upcast anything array-like (numpy, torch CPU tensor, bf16 included) to fp64."""
    if hasattr(x, "detach"):  # torch tensor: go through fp32 to leave bf16
        x = x.detach().to("cpu")
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Form 1: the definition, one query row at a time.
# ---------------------------------------------------------------------------

def softmax_row(q, K, scale):
    """Softmax weights of one query over a key set, and their log-sum-exp.

    w_j = exp(a_j - max a) / sum_l exp(a_l - max a),  a_j = scale * q.k_j
    (news.chathome.org, "What is Parallax": softmax attention as the
    Nadaraya-Watson estimator; gist.science, "Problem definition").
    Returns (w, lse) with lse = max a + ln sum exp(a - max a).
    """
    a = scale * (K @ q)
    amax = a.max()
    e = np.exp(a - amax)
    z = e.sum()
    return e / z, amax + np.log(z)


def parallax_row_explicit(q, rho, K, V, scale):
    """Parallax output for one query row by the definition.

    o = o_bar - Sigma_KV rho with Sigma_KV = sum_j w_j (v_j - o_bar)(k_j - k_bar)^T
    (gist.science, "Method: Parallax / Core mechanism", output equation;
    eta = 0 per the same section's "removing boundary amplification").

    K: [n, d_k], V: [n, d_v], q and rho: [d_k].  n == 0 gives (0, -inf).
    """
    n = K.shape[0]
    if n == 0:
        return np.zeros(V.shape[1]), -np.inf
    w, lse = softmax_row(q, K, scale)
    k_bar = w @ K                        # weighted key mean       [d_k]
    o_bar = w @ V                        # softmax output o^SA     [d_v]
    dK = K - k_bar                       # centred keys            [n, d_k]
    dV = V - o_bar                       # centred values          [n, d_v]
    sigma = dV.T @ (w[:, None] * dK)     # Sigma_KV                [d_v, d_k]
    return o_bar - sigma @ rho, lse


def _kv_head(h, Hq, Hkv):
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def _prefill_keys(i, N, causal):
    return i + 1 if causal else N


def prefill_rows_explicit(q, k, v, r, rows, causal=True, scale=None):
    """Explicit-form prefill outputs for a list of (b, h, i) rows.

    q, r: [B, Hq, N, d]; k, v: [B, Hkv, N, d] (any array-like, upcast to fp64).
    r may be None (rho = 0). Returns (o [len(rows), d], lse [len(rows)]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    r = None if r is None else _f64(r)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((len(rows), v.shape[-1]))
    lse = np.zeros(len(rows))
    for t, (b, h, i) in enumerate(rows):
        g = _kv_head(h, Hq, Hkv)
        n = _prefill_keys(i, N, causal)
        rho = np.zeros(d) if r is None else r[b, h, i]
        o[t], lse[t] = parallax_row_explicit(q[b, h, i], rho, k[b, g, :n], v[b, g, :n], scale)
    return o, lse


def prefill_explicit(q, k, v, r, causal=True, scale=None):
    """Explicit-form prefill over every row: (out [B, Hq, N, d], lse [B, Hq, N])."""
    q = _f64(q)
    B, Hq, N, _ = q.shape
    rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N)]
    o, lse = prefill_rows_explicit(q, k, v, r, rows, causal, scale)
    return o.reshape(B, Hq, N, -1), lse.reshape(B, Hq, N)


def decode_rows_explicit(q, r, kcache, vcache, seqlens, rows, scale=None):
    """Explicit-form decode outputs for a list of (b, h) rows.

    q, r: [B, Hq, d]; kcache, vcache: [B, Hkv, S_max, d]; seqlens: [B] ints.
    Query (b, h) attends the cached keys j < seqlens[b] of KV head h // G.
    """
    q, kc, vc = _f64(q), _f64(kcache), _f64(vcache)
    r = None if r is None else _f64(r)
    seqlens = np.asarray(_f64(seqlens), dtype=np.int64)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((len(rows), vc.shape[-1]))
    lse = np.zeros(len(rows))
    for t, (b, h) in enumerate(rows):
        g = _kv_head(h, Hq, Hkv)
        n = max(int(seqlens[b]), 0)
        rho = np.zeros(d) if r is None else r[b, h]
        o[t], lse[t] = parallax_row_explicit(q[b, h], rho, kc[b, g, :n], vc[b, g, :n], scale)
    return o, lse


def decode_explicit(q, r, kcache, vcache, seqlens, scale=None):
    """Explicit-form decode over every (b, h): (out [B, Hq, d], lse [B, Hq])."""
    q = _f64(q)
    B, Hq, _ = q.shape
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o, lse = decode_rows_explicit(q, r, kcache, vcache, seqlens, rows, scale)
    return o.reshape(B, Hq, -1), lse.reshape(B, Hq)


# ---------------------------------------------------------------------------
# Form 2: effective weights, one (b, head) block at a time as matrices.
# ---------------------------------------------------------------------------

def _effective_block(Q, R, K, V, mask, scale):
    """o_i = sum_j w_ij (1 - (s_ij - s_bar_i)) v_j for a block of queries.

    Q, R: [m, d]; K, V: [n, d]; mask: [m, n] bool (True = key j is in row i's
    set). Rows with an empty set give o = 0, lse = -inf.
    """
    if K.shape[0] == 0:
        return np.zeros((Q.shape[0], V.shape[1])), np.full(Q.shape[0], -np.inf)
    A = scale * (Q @ K.T)
    A = np.where(mask, A, -np.inf)
    amax = A.max(axis=1, keepdims=True)
    empty = ~np.isfinite(amax[:, 0])
    amax = np.where(np.isfinite(amax), amax, 0.0)
    E = np.where(mask, np.exp(A - amax), 0.0)
    z = E.sum(axis=1, keepdims=True)
    zsafe = np.where(z > 0, z, 1.0)
    W = E / zsafe
    if R is None:
        W_hat = W
    else:
        S = R @ K.T
        s_bar = (W * S).sum(axis=1, keepdims=True)
        W_hat = W * (1.0 - (S - s_bar))
    O = W_hat @ V
    lse = amax[:, 0] + np.log(zsafe[:, 0])
    O[empty] = 0.0
    lse[empty] = -np.inf
    return O, lse


def prefill_effective(q, k, v, r, causal=True, scale=None, heads=None):
    """Effective-weight prefill. heads: optional list of (b, h) to compute
    (the rest is left NaN). Returns (out [B, Hq, N, d], lse [B, Hq, N])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    r = None if r is None else _f64(r)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, N, v.shape[-1]), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    ii = np.arange(N)[:, None]
    jj = np.arange(N)[None, :]
    mask = (jj <= ii) if causal else np.ones((N, N), dtype=bool)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in heads:
        g = _kv_head(h, Hq, Hkv)
        R = None if r is None else r[b, h]
        out[b, h], lse[b, h] = _effective_block(q[b, h], R, k[b, g], v[b, g], mask, scale)
    return out, lse


def decode_effective(q, r, kcache, vcache, seqlens, scale=None, batches=None):
    """Effective-weight decode. batches: optional list of b to compute (rest NaN).
    Returns (out [B, Hq, d], lse [B, Hq])."""
    q, kc, vc = _f64(q), _f64(kcache), _f64(vcache)
    r = None if r is None else _f64(r)
    seqlens = np.asarray(_f64(seqlens), dtype=np.int64)
    B, Hq, d = q.shape
    Hkv, S_max = kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, vc.shape[-1]), np.nan)
    lse = np.full((B, Hq), np.nan)
    if batches is None:
        batches = range(B)
    for b in batches:
        n = min(max(int(seqlens[b]), 0), S_max)
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            mask = np.ones((G, n), dtype=bool)
            R = None if r is None else r[b, hs]
            out[b, hs], lse[b, hs] = _effective_block(q[b, hs], R, kc[b, g, :n], vc[b, g, :n], mask, scale)
    return out, lse
