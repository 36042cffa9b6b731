"""Pins for the streamed form of the fp64 oracle: checks against what the pages
and the mathematics fix, never against the form itself.

The streamed form is the one of news.chathome.org, "Parallax: a parameterized
local linear attention ...", section "Hardware argument": two score branches
sharing the online maximum, accumulating (m, l, c, O1, O2) and emitting
O1/l - (O2/l - (c/l)(O1/l)). The pins:
- the row pins of the explicit and effective forms (hand-derived examples,
  rho = 0 against SDPA, the two-key closed form, one key, identical keys,
  linearity in rho, translations, permutations, the value-by-key
  orientation), for chunks of 1 key, 3 keys and all keys;
- brute force on tiny inputs: every partition of the keys into disjoint
  sets, merged in any order or as a tree, gives the explicit definition's
  output and lse;
- the reference maximum of a merge is free: rescaling both states to any
  common reference gives the same result (the freedom a lazy rescale uses);
- merging with an empty set changes nothing; an empty key set gives o = 0
  and lse = -inf;
- planted mistakes in copies of the streamed row (a term left unrescaled,
  no rescale at all, lse without the maximum, c from unweighted scores) are
  each rejected.
"""
import math

import numpy as np
import pytest

import oracle
import test_oracle_pins as P
from oracle import plx_oracle_stream as S

RNG = np.random.default_rng(4321)


@pytest.mark.parametrize("chunk", [None, 1, 3])
@pytest.mark.parametrize("pin", P.ROW_PINS, ids=lambda f: f.__name__)
def test_row_pins_streamed_form(pin, chunk):
    pin(lambda q, rho, K, V, scale: S.parallax_row_streamed(q, rho, K, V, scale, chunk))


def _row(n, d=5, spread=3.0):
    """A row whose scores span several units, so that chunk maxima differ."""
    q = RNG.standard_normal(d) * spread
    return q, RNG.standard_normal(d) * 0.7, RNG.standard_normal((n, d)), RNG.standard_normal((n, d))


def _close(o, lse, ref_o, ref_lse):
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-10)
    assert abs(lse - ref_lse) < 1e-10


def test_any_partition_and_order_matches_explicit():
    for _ in range(40):
        n = int(RNG.integers(1, 30))
        q, rho, K, V = _row(n)
        scale = 0.45
        idx = RNG.permutation(n)
        cuts = np.sort(RNG.choice(np.arange(1, n), size=min(n - 1, int(RNG.integers(0, 6))), replace=False)) if n > 1 else []
        parts = np.split(idx, cuts)
        states = [S.chunk_state(q, rho, K[p], V[p], scale) for p in parts]
        ref = oracle.parallax_row_explicit(q, rho, K, V, scale)
        st = S.empty_state(V.shape[1])
        for i in RNG.permutation(len(states)):
            st = S.merge_states(st, states[i])
        _close(*S.finish_state(st), *ref)
        # as a tree: pairwise merges, level by level
        level = list(states)
        while len(level) > 1:
            level = [S.merge_states(level[i], level[i + 1]) if i + 1 < len(level) else level[i]
                     for i in range(0, len(level), 2)]
        _close(*S.finish_state(level[0]), *ref)


@pytest.mark.parametrize("chunk", [1, 2, 5, 64])
def test_streamed_row_equals_explicit(chunk):
    for n in (1, 2, 7, 33):
        q, rho, K, V = _row(n, d=8)
        _close(*S.parallax_row_streamed(q, rho, K, V, 0.35, chunk), *oracle.parallax_row_explicit(q, rho, K, V, 0.35))


def test_reference_maximum_is_free():
    """Rescaling both states to any common reference t (not only the larger
    maximum) and adding gives the same result: l, c, O1, O2 all carry the same
    factor exp(m - t), which the finishing divisions cancel."""
    q, rho, K, V = _row(12)
    a_state = S.chunk_state(q, rho, K[:5], V[:5], 0.5)
    b_state = S.chunk_state(q, rho, K[5:], V[5:], 0.5)
    ref = S.finish_state(S.merge_states(a_state, b_state))
    for t in (a_state[0], b_state[0], max(a_state[0], b_state[0]) + 3.0, min(a_state[0], b_state[0]) - 2.0):
        f1, f2 = math.exp(a_state[0] - t), math.exp(b_state[0] - t)
        st = (t,) + tuple(f1 * x + f2 * y for x, y in zip(a_state[1:], b_state[1:]))
        _close(*S.finish_state(st), *ref)


def test_empty_sets():
    q, rho, K, V = _row(6)
    x = S.chunk_state(q, rho, K, V, 0.5)
    e = S.empty_state(V.shape[1])
    for st in (S.merge_states(e, x), S.merge_states(x, e)):
        assert st[0] == x[0] and st[1] == x[1] and st[2] == x[2]
        np.testing.assert_array_equal(st[3], x[3])
        np.testing.assert_array_equal(st[4], x[4])
    o, lse = S.finish_state(S.merge_states(e, e))
    assert lse == -np.inf and not o.any()
    o, lse = S.parallax_row_streamed(q, rho, K[:0], V[:0], 0.5, 2)
    ro, rl = oracle.parallax_row_explicit(q, rho, K[:0], V[:0], 0.5)
    np.testing.assert_array_equal(o, ro)
    assert lse == rl == -np.inf


# ---------------------------------------------------------------------------
# Mutants: plausible slips planted in copies of the streamed row.
# ---------------------------------------------------------------------------

def _mutant(kind):
    def state(q, rho, K, V, scale):
        a = scale * (K @ q)
        s = K @ rho
        m = a.max()
        p = np.exp(a - m)
        c = s.sum() if kind == "c_unweighted" else (p * s).sum()
        return m, p.sum(), c, p @ V, (p * s) @ V

    def merge(x, y):
        m1, l1, c1, a1, b1 = x
        m2, l2, c2, a2, b2 = y
        m = max(m1, m2)
        f1 = 0.0 if m1 == -np.inf else math.exp(m1 - m)
        f2 = 0.0 if m2 == -np.inf else math.exp(m2 - m)
        if kind == "no_rescale":
            f1 = f2 = 1.0
        c = c1 + c2 if kind == "c_unrescaled" else f1 * c1 + f2 * c2
        O2 = b1 + b2 if kind == "o2_unrescaled" else f1 * b1 + f2 * b2
        return m, f1 * l1 + f2 * l2, c, f1 * a1 + f2 * a2, O2

    def row(q, rho, K, V, scale):
        st = (-np.inf, 0.0, 0.0, np.zeros(V.shape[1]), np.zeros(V.shape[1]))
        for j0 in range(0, K.shape[0], 3):
            st = merge(st, state(q, rho, K[j0:j0 + 3], V[j0:j0 + 3], scale))
        m, l, c, O1, O2 = st
        o1 = O1 / l
        lse = math.log(l) if kind == "lse_without_max" else m + math.log(l)
        return o1 - (O2 / l - (c / l) * o1), lse

    return row


MUTANTS = ["c_unrescaled", "o2_unrescaled", "no_rescale", "lse_without_max", "c_unweighted"]


def _battery(row):
    """The row pins plus a brute-force comparison on rows whose chunk maxima differ."""
    failures = 0
    for pin in P.ROW_PINS:
        try:
            pin(row)
        except (AssertionError, OverflowError, FloatingPointError, ValueError, ZeroDivisionError):
            failures += 1
    for n in (4, 9, 17):
        q, rho, K, V = _row(n)
        try:
            _close(*row(q, rho, K, V, 0.5), *oracle.parallax_row_explicit(q, rho, K, V, 0.5))
        except AssertionError:
            failures += 1
    return failures


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutants_are_caught(kind):
    assert _battery(_mutant(kind)) > 0, f"no pin rejects the {kind} mutant"


def test_unmutated_copy_passes():
    assert _battery(_mutant("none")) == 0
