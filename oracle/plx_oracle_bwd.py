"""Plain fp64 CPU oracle for the gradients of the Parallax attention forward.

THIS IS TEST INFRASTRUCTURE, under the same rule as ``plx_oracle``: only the
tests, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may use
it, and it shares nothing with the library.

The pages give the forward only (gist.science, "Technical overview: Parallax
- parameterized local linear attention for language modeling", section
"Method: Parallax / Core mechanism": o_i = o^SA_i - Sigma^(i)_KV rho_i with
eta = 0), and say the method is trained end to end as a pretraining
architecture (same page, "Experimental setup"; news.chathome.org, "Parallax:
a parameterized local linear attention ...", section "Training").  The
gradients here are those of that forward with respect to q, k, v and rho,
for the loss L = sum_i dO_i . o_i.

Two independent forms:

1. ``prefill_backward_autograd``: reverse-mode differentiation (torch
   autograd, fp64, CPU) of the forward written out by its definition, with the
   explicit d x d matrix Sigma_KV per query row.  Nothing about the gradient
   is derived by hand.  Cost ~ N^2 d^2 per head: small inputs only.

2. ``prefill_backward_closed``: the gradient derived by hand from the
   effective-weight form of the forward (o_i = sum_j w_ij (1 - s_ij + s_bar_i) v_j,
   s_ij = rho_i . k_j, s_bar_i = sum_j w_ij s_ij; the covariance identity
   that gives this form is stated in ``plx_oracle``).  With g_ij = dO_i . v_j,
   g_bar_i = sum_j w_ij g_ij and D_i = dO_i . o_i + s_bar_i g_bar_i:

       dV_j  = sum_i w_hat_ij dO_i,          w_hat_ij = w_ij (1 - s_ij + s_bar_i)
       dS_ij = w_ij (g_bar_i - g_ij)                      (d L / d s_ij)
       dA_ij = w_ij (g_ij (1 - s_ij + s_bar_i) + s_ij g_bar_i - D_i)   (d L / d a_ij)
       dQ_i  = scale sum_j dA_ij k_j
       dK_j  = scale sum_i dA_ij q_i + sum_i dS_ij rho_i
       dR_i  = sum_j dS_ij k_j

   (a_ij = scale q_i . k_j; w = softmax_j(a)).  The derivation: with
   A = sum_l w_l v_l and s_bar = sum_l w_l s_l, o = A - sum_l w_l s_l v_l + s_bar A,
   so d o / d w_j = (1 - s_j + s_bar) v_j + s_j o_bar and
   d o / d s_j = w_j (o_bar - v_j); the softmax Jacobian then gives dA with
   sum_l w_l (dL/dw_l) = dO . o + s_bar g_bar.  Whole (b, head) blocks as
   N x N matrices: used for full heads at large sizes.

The tests pin form 2 against form 1, against central finite differences of
the numpy forward oracle, against softmax attention's gradients at rho = 0
(the pages: probe norm zero reduces to softmax attention), and against the
invariants sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 (shifting every key or
every value by one vector leaves the weights unchanged).

``prefill_aux`` gives the two per-row quantities a training forward keeps for
the backward: o_bar_i = sum_j w_ij v_j (the softmax output) and s_bar_i.
"""
from __future__ import annotations

import numpy as np

from .plx_oracle import _f64, _kv_head

__all__ = [
    "prefill_backward_autograd",
    "prefill_backward_closed",
    "prefill_aux",
]


def _mask(N, causal):
    ii = np.arange(N)[:, None]
    jj = np.arange(N)[None, :]
    return (jj <= ii) if causal else np.ones((N, N), dtype=bool)


def _softmax_masked(A, mask):
    A = np.where(mask, A, -np.inf)
    amax = A.max(axis=1, keepdims=True)
    E = np.where(mask, np.exp(A - amax), 0.0)
    return E / E.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# Form 1: autograd through the definition (explicit Sigma_KV per row).
# ---------------------------------------------------------------------------

def _explicit_block_torch(torch, Q, R, K, V, mask, scale):
    A = scale * (Q @ K.T)
    A = A.masked_fill(~mask, float("-inf"))
    W = torch.softmax(A, dim=1)
    k_bar = W @ K                                   # [m, d]
    o_bar = W @ V                                   # [m, d]
    Vc = V[None, :, :] - o_bar[:, None, :]          # v_j - o_bar_i   [m, n, d]
    Kc = K[None, :, :] - k_bar[:, None, :]          # k_j - k_bar_i   [m, n, d]
    sigma = torch.einsum("ij,ijd,ije->ide", W, Vc, Kc)   # Sigma_KV per row [m, d_v, d_k]
    return o_bar - torch.einsum("ide,ie->id", sigma, R)


def prefill_backward_autograd(q, k, v, r, do, causal=True, scale=None):
    """Gradients (dq, dk, dv, dr) of L = sum dO . o by torch autograd of the
    explicit definition.  q, r, do: [B, Hq, N, d]; k, v: [B, Hkv, N, d];
    r None means rho = 0 (dr is still returned: the gradient at rho = 0)."""
    import torch

    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    r = np.zeros_like(q) if r is None else _f64(r)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    mask = torch.from_numpy(_mask(N, causal))
    dq, dr = np.zeros_like(q), np.zeros_like(r)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            Q = torch.tensor(q[b, h], dtype=torch.float64, requires_grad=True)
            R = torch.tensor(r[b, h], dtype=torch.float64, requires_grad=True)
            K = torch.tensor(k[b, g], dtype=torch.float64, requires_grad=True)
            V = torch.tensor(v[b, g], dtype=torch.float64, requires_grad=True)
            O = _explicit_block_torch(torch, Q, R, K, V, mask, scale)
            loss = (O * torch.from_numpy(do[b, h])).sum()
            gq, gk, gv, gr = torch.autograd.grad(loss, (Q, K, V, R))
            dq[b, h] = gq.numpy()
            dr[b, h] = gr.numpy()
            dk[b, g] += gk.numpy()
            dv[b, g] += gv.numpy()
    return dq, dk, dv, dr


# ---------------------------------------------------------------------------
# Form 2: the closed-form gradient, whole heads as matrices.
# ---------------------------------------------------------------------------

def _closed_block(Q, R, K, V, dO, mask, scale):
    W = _softmax_masked(scale * (Q @ K.T), mask)
    S = R @ K.T
    G = dO @ V.T
    s_bar = (W * S).sum(axis=1, keepdims=True)
    g_bar = (W * G).sum(axis=1, keepdims=True)
    W_hat = W * (1.0 - S + s_bar)
    O = W_hat @ V
    D = (dO * O).sum(axis=1, keepdims=True) + s_bar * g_bar
    dS = W * (g_bar - G)
    dA = W * (G * (1.0 - S + s_bar) + S * g_bar - D)
    return scale * (dA @ K), scale * (dA.T @ Q) + dS.T @ R, W_hat.T @ dO, dS @ K


def prefill_backward_closed(q, k, v, r, do, causal=True, scale=None, heads=None):
    """Closed-form gradients (dq, dk, dv, dr).  heads: optional list of (b, h)
    query heads to include; dq / dr of other heads are NaN and dk / dv then
    hold only the listed heads' contributions."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    r = np.zeros_like(q) if r is None else _f64(r)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    mask = _mask(N, causal)
    dq, dr = np.full_like(q, np.nan), np.full_like(r, np.nan)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in heads:
        g = _kv_head(h, Hq, Hkv)
        gq, gk, gv, gr = _closed_block(q[b, h], r[b, h], k[b, g], v[b, g], do[b, h], mask, scale)
        dq[b, h], dr[b, h] = gq, gr
        dk[b, g] += gk
        dv[b, g] += gv
    return dq, dk, dv, dr


def prefill_aux(q, k, v, r, causal=True, scale=None, heads=None):
    """Per-row o_bar = sum_j w_ij v_j [B, Hq, N, d] and s_bar = sum_j w_ij s_ij
    [B, Hq, N] (s_bar = 0 when r is None).  heads as in prefill_backward_closed."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    r = np.zeros_like(q) if r is None else _f64(r)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    mask = _mask(N, causal)
    o_bar = np.full((B, Hq, N, v.shape[-1]), np.nan)
    s_bar = np.full((B, Hq, N), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in heads:
        g = _kv_head(h, Hq, Hkv)
        W = _softmax_masked(scale * (q[b, h] @ k[b, g].T), mask)
        o_bar[b, h] = W @ v[b, g]
        s_bar[b, h] = (W * (r[b, h] @ k[b, g].T)).sum(axis=1)
    return o_bar, s_bar
