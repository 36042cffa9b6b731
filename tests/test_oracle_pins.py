"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

Formula: gist.science, "Technical overview: Parallax - parameterized local
linear attention for language modeling", section "Method: Parallax / Core
mechanism" (o = o_SA - Sigma_KV rho, eta = 0). Special case rho = 0 is exactly
softmax attention: news.chathome.org, "Parallax: a parameterized local linear
attention ...", section "How the mechanism works" (probe norm zero).

Each check below is chosen so that a plausible slip in the oracle (a sign, a
transposed Sigma, a missing centring, a Bessel factor, a scaled rho branch,
an off-by-one causal set, a wrong GQA head) fails at least one of them;
``test_mutants_are_caught`` plants such slips in copies of the oracle's row
function and checks that the battery rejects every one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
RNG = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# Row-level pins, parameterised over an implementation so mutants can be run.
# ---------------------------------------------------------------------------

def pin_golden(row_fn):
    """Hand-derived exact examples (tests/golden/hand_examples.json)."""
    ex = json.load(open(GOLDEN))["examples"]
    for e in ex:
        o, lse = row_fn(np.array(e["q"]), np.array(e["rho"]), np.array(e["K"]),
                        np.array(e["V"]), e["scale"])
        np.testing.assert_allclose(o, e["expected_o"], rtol=0, atol=1e-12, err_msg=e["name"])
        assert abs(lse - e["expected_lse"]) < 1e-12, e["name"]


def pin_rho_zero_is_softmax(row_fn):
    """rho = 0: o = sum_j softmax_j v_j, checked against torch SDPA (fp64)."""
    d, n = 8, 13
    q, K, V = _rand(d), _rand(n, d), _rand(n, d)
    scale = 1 / math.sqrt(d)
    o, lse = row_fn(q, np.zeros(d), K, V, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None, None], torch.tensor(K)[None, None],
        torch.tensor(V)[None, None], scale=scale)[0, 0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    assert abs(lse - scipy.special.logsumexp(scale * K @ q)) < 1e-12


def pin_two_key_closed_form(row_fn):
    """Two keys: Sigma rho = w0 w1 (v1 - v0) (rho.(k1 - k0)) exactly."""
    d = 5
    q, rho = _rand(d), _rand(d)
    K, V = _rand(2, d), _rand(2, d)
    scale = 0.7
    a = scale * K @ q
    w1 = 1.0 / (1.0 + math.exp(a[0] - a[1]))
    w0 = 1.0 - w1
    o_sa = w0 * V[0] + w1 * V[1]
    expect = o_sa - w0 * w1 * (V[1] - V[0]) * float(rho @ (K[1] - K[0]))
    o, lse = row_fn(q, rho, K, V, scale)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-12)
    assert abs(lse - (max(a) + math.log1p(math.exp(-abs(a[0] - a[1]))))) < 1e-12


def pin_single_key(row_fn):
    """One key: Sigma = 0, o = v0 for any q, rho."""
    d = 6
    o, lse = row_fn(_rand(d), _rand(d, scale=5), _rand(1, d), V := _rand(1, d), 0.3)
    np.testing.assert_allclose(o, V[0], rtol=0, atol=1e-13)


def pin_identical_keys(row_fn):
    """Identical keys: uniform weights, zero correction, o = mean(V),
    lse = scale q.k + ln n."""
    d, n = 4, 7
    q, k = _rand(d), _rand(d)
    K = np.tile(k, (n, 1))
    V = _rand(n, d)
    o, lse = row_fn(q, _rand(d, scale=3), K, V, 0.5)
    np.testing.assert_allclose(o, V.mean(0), rtol=0, atol=1e-12)
    assert abs(lse - (0.5 * float(q @ k) + math.log(n))) < 1e-12


def pin_linear_in_rho(row_fn):
    """o(a r1 + b r2) - o_SA = a (o(r1) - o_SA) + b (o(r2) - o_SA)."""
    d, n = 6, 9
    q, K, V = _rand(d), _rand(n, d), _rand(n, d)
    r1, r2 = _rand(d), _rand(d)
    o_sa, _ = row_fn(q, np.zeros(d), K, V, 0.4)
    o1, _ = row_fn(q, r1, K, V, 0.4)
    o2, _ = row_fn(q, r2, K, V, 0.4)
    o12, _ = row_fn(q, 2.5 * r1 - 1.5 * r2, K, V, 0.4)
    np.testing.assert_allclose(o12 - o_sa, 2.5 * (o1 - o_sa) - 1.5 * (o2 - o_sa), rtol=0, atol=1e-11)


def pin_translations(row_fn):
    """k -> k + t: o unchanged, lse shifts by scale q.t; v -> v + t: o shifts by t."""
    d, n = 5, 11
    q, rho, K, V, t = _rand(d), _rand(d), _rand(n, d), _rand(n, d), _rand(d)
    o, lse = row_fn(q, rho, K, V, 0.6)
    o_k, lse_k = row_fn(q, rho, K + t, V, 0.6)
    o_v, lse_v = row_fn(q, rho, K, V + t, 0.6)
    np.testing.assert_allclose(o_k, o, rtol=0, atol=1e-11)
    assert abs(lse_k - (lse + 0.6 * float(q @ t))) < 1e-11
    np.testing.assert_allclose(o_v, o + t, rtol=0, atol=1e-11)
    assert abs(lse_v - lse) < 1e-13


def pin_permutation(row_fn):
    """Joint permutation of (k_j, v_j) leaves the result unchanged."""
    d, n = 4, 10
    q, rho, K, V = _rand(d), _rand(d), _rand(n, d), _rand(n, d)
    p = RNG.permutation(n)
    o, lse = row_fn(q, rho, K, V, 0.5)
    o_p, lse_p = row_fn(q, rho, K[p], V[p], 0.5)
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-12)
    assert abs(lse_p - lse) < 1e-12


def pin_asymmetric_orientation(row_fn):
    """Sigma is value-by-key: with d_v != d_k the product Sigma rho must be a
    value-space vector; keys in 3-d, values in 2-d."""
    q, rho, K, V = _rand(3), _rand(3), _rand(2, 3), _rand(2, 2)
    a = 0.5 * K @ q
    w1 = 1.0 / (1.0 + math.exp(a[0] - a[1]))
    w0 = 1.0 - w1
    expect = w0 * V[0] + w1 * V[1] - w0 * w1 * (V[1] - V[0]) * float(rho @ (K[1] - K[0]))
    o, _ = row_fn(q, rho, K, V, 0.5)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-12)


ROW_PINS = [pin_golden, pin_rho_zero_is_softmax, pin_two_key_closed_form, pin_single_key,
            pin_identical_keys, pin_linear_in_rho, pin_translations, pin_permutation,
            pin_asymmetric_orientation]


@pytest.mark.parametrize("pin", ROW_PINS, ids=lambda f: f.__name__)
def test_row_pins(pin):
    pin(oracle.parallax_row_explicit)


def _effective_row(q, rho, K, V, scale):
    """The oracle's effective-weight block path on a single row."""
    mask = np.ones((1, K.shape[0]), dtype=bool)
    o, lse = oracle.plx_oracle._effective_block(q[None], rho[None], K, V, mask, scale)
    return o[0], lse[0]


@pytest.mark.parametrize("pin", ROW_PINS, ids=lambda f: f.__name__)
def test_row_pins_effective_form(pin):
    pin(_effective_row)


# ---------------------------------------------------------------------------
# Mutants: plausible slips planted in copies of the row function.
# ---------------------------------------------------------------------------

def _mutant(kind):
    def row(q, rho, K, V, scale):
        a = scale * (K @ q)
        e = np.exp(a - a.max())
        w = e / e.sum()
        lse = a.max() + math.log(e.sum())
        if kind == "lse_log2":
            lse = a.max() + math.log2(e.sum())
        kb, ob = w @ K, w @ V
        if kind == "uniform_centre":
            kb, ob = K.mean(0), V.mean(0)
        dK, dV = K - kb, V - ob
        if kind == "no_centring":
            dK, dV = K, V
        ww = w
        if kind == "uniform_cov_weights":
            ww = np.full_like(w, 1.0 / len(w))
        sigma = dV.T @ (ww[:, None] * dK)
        if kind == "bessel":
            sigma = sigma * len(w) / max(len(w) - 1, 1)
        if kind == "transposed":  # key-by-value instead of value-by-key
            sigma = dK.T @ (ww[:, None] * dV)
        r = rho * (scale if kind == "scaled_rho" else 1.0)
        sign = 1.0 if kind == "plus_sign" else -1.0
        o = ob + sign * (sigma @ r)
        if kind == "eta_term":
            o = o + (ob - ob.mean())  # a spurious extra term
        if kind == "scale_missing":
            a2 = K @ q
            e2 = np.exp(a2 - a2.max())
            w2 = e2 / e2.sum()
            o = w2 @ V - (V - w2 @ V).T @ (w2[:, None] * (K - w2 @ K)) @ rho
        return o, lse
    return row


MUTANTS = ["plus_sign", "transposed", "no_centring", "uniform_centre", "uniform_cov_weights",
           "bessel", "scaled_rho", "eta_term", "scale_missing", "lse_log2"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutants_are_caught(kind):
    row = _mutant(kind)
    failures = 0
    for pin in ROW_PINS:
        try:
            pin(row)
        except (AssertionError, OverflowError, FloatingPointError, ValueError):
            failures += 1
    assert failures > 0, f"no pin rejects the {kind} mutant"


def test_unmutated_copy_passes():
    row = _mutant("none")
    for pin in ROW_PINS:
        pin(row)


# ---------------------------------------------------------------------------
# Tensor-level pins: causal sets, GQA mapping, decode, the two forms.
# ---------------------------------------------------------------------------

def _prefill(B=2, Hq=4, Hkv=2, N=17, d=8, rs=0.3):
    return (_rand(B, Hq, N, d), _rand(B, Hkv, N, d), _rand(B, Hkv, N, d), _rand(B, Hq, N, d, scale=rs))


@pytest.mark.parametrize("N,d", [(1, 4), (2, 4), (3, 8), (17, 8), (33, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_explicit_equals_effective(N, d, causal):
    q, k, v, r = _prefill(B=1, Hq=2, Hkv=1, N=N, d=d)
    o1, l1 = oracle.prefill_explicit(q, k, v, r, causal)
    o2, l2 = oracle.prefill_effective(q, k, v, r, causal)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_rho_zero_prefill_matches_sdpa_gqa_causal():
    q, k, v, _ = _prefill(B=2, Hq=4, Hkv=2, N=19, d=8)
    o, lse = oracle.prefill_effective(q, k, v, None, True)
    G = 2
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k).repeat_interleave(G, 1),
        torch.tensor(v).repeat_interleave(G, 1), is_causal=True).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    s = np.einsum("bhid,bhjd->bhij", q, np.repeat(k, G, 1)) / math.sqrt(8)
    s = np.where(np.tril(np.ones((19, 19), bool)), s, -np.inf)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_causal_row_is_prefix_attention():
    """Causal row i equals a non-causal problem over keys 0..i (diagonal included)."""
    q, k, v, r = _prefill(B=1, Hq=1, Hkv=1, N=9, d=4)
    o, lse = oracle.prefill_explicit(q, k, v, r, True)
    for i in range(9):
        oi, li = oracle.parallax_row_explicit(q[0, 0, i], r[0, 0, i], k[0, 0, : i + 1], v[0, 0, : i + 1], 0.5)
        np.testing.assert_allclose(o[0, 0, i], oi, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], rtol=0, atol=1e-13)  # one key: v0


def test_gqa_equals_repeated_mha():
    q, k, v, r = _prefill(B=1, Hq=6, Hkv=2, N=11, d=8)
    o, lse = oracle.prefill_effective(q, k, v, r, True)
    o_m, lse_m = oracle.prefill_effective(q, np.repeat(k, 3, 1), np.repeat(v, 3, 1), r, True)
    np.testing.assert_allclose(o, o_m, rtol=0, atol=0)
    # head h must read KV head h // 3: swapping KV heads changes heads 0..2 only
    o_s, _ = oracle.prefill_effective(q, k[:, ::-1].copy(), v[:, ::-1].copy(), r, True)
    assert not np.allclose(o_s[:, :3], o[:, :3])
    o_h1, _ = oracle.prefill_effective(q[:, :3], k[:, 1:2], v[:, 1:2], r[:, :3], True)
    np.testing.assert_allclose(o_s[:, :3], o_h1, rtol=0, atol=0)


def test_decode_is_last_prefill_row_and_empty_context():
    B, Hq, Hkv, S, d = 3, 4, 2, 12, 8
    q, kc, vc, r = _rand(B, Hq, d), _rand(B, Hkv, S, d), _rand(B, Hkv, S, d), _rand(B, Hq, d, scale=0.3)
    seqlens = np.array([12, 5, 0])
    o_e, l_e = oracle.decode_explicit(q, r, kc, vc, seqlens)
    o_w, l_w = oracle.decode_effective(q, r, kc, vc, seqlens)
    np.testing.assert_allclose(o_e, o_w, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_e[:2], l_w[:2], rtol=0, atol=1e-12)
    assert np.all(o_e[2] == 0) and np.all(np.isneginf(l_e[2])) and np.all(np.isneginf(l_w[2]))
    # decode row with seqlen n == causal prefill row n-1 with q, r placed there
    for b, n in [(0, 12), (1, 5)]:
        Q = np.zeros((1, Hq, n, d)); Q[0, :, n - 1] = q[b]
        R = np.zeros((1, Hq, n, d)); R[0, :, n - 1] = r[b]
        o_p, l_p = oracle.prefill_effective(Q, kc[b:b + 1, :, :n], vc[b:b + 1, :, :n], R, True)
        np.testing.assert_allclose(o_p[0, :, n - 1], o_e[b], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l_p[0, :, n - 1], l_e[b], rtol=0, atol=1e-12)


def test_effective_weights_sum_to_one_and_can_be_negative():
    """The effective weights w(1 - (s - s_bar)) sum to 1; with a large probe
    some are negative or exceed 1 (news.chathome.org, 'Score differences')."""
    d, n = 8, 50
    q, rho, K = _rand(d), _rand(d, scale=2.0), _rand(n, d)
    # with V = identity the output is the effective weight vector itself
    o, _ = oracle.parallax_row_explicit(q, rho, K, np.eye(n), 1 / math.sqrt(d))
    assert abs(o.sum() - 1.0) < 1e-12
    assert (o < 0).any() or (o > 1).any()


def test_bf16_inputs_upcast_exactly():
    t = torch.randn(2, 1, 3, 4).to(torch.bfloat16)
    x = oracle.plx_oracle._f64(t)
    assert x.dtype == np.float64
    np.testing.assert_array_equal(x, t.float().numpy().astype(np.float64))
