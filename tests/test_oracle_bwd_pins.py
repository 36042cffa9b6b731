"""Pins of the gradient oracle to things other than itself (CPU, fp64)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import plx_oracle_bwd as ob
from parameterized_local_linear_plx_b200 import inputs


def _case(B, Hq, Hkv, N, d, seed, r_scale=0.3):
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=seed, r_scale=r_scale, dtype=torch.float32)
    g = torch.Generator().manual_seed(seed + 1000)
    do = torch.randn(q.shape, generator=g)
    return [t.double().numpy() for t in (q, k, v, r, do)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2)])
def test_closed_form_equals_autograd_of_definition(causal, Hq, Hkv):
    """Hand-derived gradient == reverse-mode derivative of the explicit-Sigma forward."""
    q, k, v, r, do = _case(1, Hq, Hkv, 23, 8, seed=5 + Hq)
    a = oracle.prefill_backward_autograd(q, k, v, r, do, causal)
    c = oracle.prefill_backward_closed(q, k, v, r, do, causal)
    for x, y, name in zip(a, c, "qkvr"):
        assert np.abs(x - y).max() <= 1e-10 * max(1.0, np.abs(x).max()), name


@pytest.mark.parametrize("causal", [True, False])
def test_closed_form_matches_finite_differences(causal):
    """Central differences of the numpy forward (effective-weight form) at
    random coordinates of q, k, v and rho, loss sum dO . o."""
    B, Hq, Hkv, N, d = 1, 2, 1, 11, 6
    q, k, v, r, do = _case(B, Hq, Hkv, N, d, seed=17)
    dq, dk, dv, dr = oracle.prefill_backward_closed(q, k, v, r, do, causal)

    def loss(q_, k_, v_, r_):
        o, _ = oracle.prefill_effective(q_, k_, v_, r_, causal)
        return float((o * do).sum())

    rng = np.random.default_rng(3)
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("r", dr)):
        args = {"q": q, "k": k, "v": v, "r": r}
        x = args[name]
        for _ in range(6):
            idx = tuple(int(rng.integers(s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            ap, am = dict(args), dict(args)
            ap[name], am[name] = xp, xm
            fd = (loss(ap["q"], ap["k"], ap["v"], ap["r"]) - loss(am["q"], am["k"], am["v"], am["r"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_rho_zero_is_softmax_attention_backward():
    """rho = 0 reduces Parallax to softmax attention (news.chathome.org, "How
    the mechanism works"), so dq, dk, dv are SDPA's gradients."""
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 8
    q, k, v, _, do = _case(B, Hq, Hkv, N, d, seed=29)
    dq, dk, dv, _ = oracle.prefill_backward_closed(q, k, v, None, do, True)
    Q = torch.tensor(q, requires_grad=True)
    K = torch.tensor(k, requires_grad=True)
    V = torch.tensor(v, requires_grad=True)
    O = torch.nn.functional.scaled_dot_product_attention(
        Q, K.repeat_interleave(Hq // Hkv, 1), V.repeat_interleave(Hq // Hkv, 1), is_causal=True)
    gq, gk, gv = torch.autograd.grad((O * torch.from_numpy(do)).sum(), (Q, K, V))
    for x, y in ((dq, gq), (dk, gk), (dv, gv)):
        assert np.abs(x - y.numpy()).max() <= 1e-12


def test_shift_invariants():
    """Adding one vector to every value adds it to every output (the
    effective weights sum to 1): sum_j dV_j = sum_i dO_i over the group.
    Adding one vector to every key shifts each row's q.k and rho.k by a
    constant: the output is unchanged, so sum_j dK_j = 0."""
    B, Hq, Hkv, N, d = 2, 4, 2, 33, 8
    q, k, v, r, do = _case(B, Hq, Hkv, N, d, seed=41, r_scale=0.5)
    _, dk, dv, _ = oracle.prefill_backward_closed(q, k, v, r, do, True)
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            want = do[b, g * G:(g + 1) * G].sum(axis=(0, 1))
            assert np.abs(dv[b, g].sum(axis=0) - want).max() <= 1e-11
            assert np.abs(dk[b, g].sum(axis=0)).max() <= 1e-11


def test_planted_mistake_is_caught():
    """A copy of the closed form without s_bar in the effective weight (a
    plausible slip) disagrees with autograd of the definition."""
    q, k, v, r, do = _case(1, 1, 1, 15, 8, seed=7, r_scale=0.5)
    mask = ob._mask(15, True)

    def wrong_block(Q, R, K, V, dO, mask, scale):
        W = ob._softmax_masked(scale * (Q @ K.T), mask)
        S = R @ K.T
        return (W * (1.0 - S)).T @ dO  # dV with s_bar dropped

    a = oracle.prefill_backward_autograd(q, k, v, r, do, True)
    bad_dv = wrong_block(q[0, 0], r[0, 0], k[0, 0], v[0, 0], do[0, 0], mask, 1 / np.sqrt(8))
    assert np.abs(bad_dv - a[2][0, 0]).max() > 1e-3


def test_aux_matches_softmax_attention_and_s_bar():
    """o_bar is softmax attention (SDPA in fp64); s_bar = rho . k_bar with
    k_bar the softmax-weighted key mean (softmax attention with V := K)."""
    B, Hq, Hkv, N, d = 1, 2, 1, 21, 8
    q, k, v, r, _ = _case(B, Hq, Hkv, N, d, seed=51)
    o_bar, s_bar = oracle.prefill_aux(q, k, v, r, True)
    t = torch.from_numpy
    sd = torch.nn.functional.scaled_dot_product_attention
    ref_o = sd(t(q), t(k).repeat_interleave(2, 1), t(v).repeat_interleave(2, 1), is_causal=True).numpy()
    k_bar = sd(t(q), t(k).repeat_interleave(2, 1), t(k).repeat_interleave(2, 1), is_causal=True).numpy()
    assert np.abs(o_bar - ref_o).max() <= 1e-12
    assert np.abs(s_bar - (k_bar * r).sum(-1)).max() <= 1e-12
