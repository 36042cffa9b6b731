"""fp64 CPU oracle: the streamed (online) form of the Parallax forward pass.

THIS IS TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py`` may import it. The
library's product path never calls anything here, and nothing here calls the
library: the two share no code, no constants and no helpers.

What it computes, and where the pages say so
--------------------------------------------
news.chathome.org, "Parallax: a parameterized local linear attention that
keeps Softmax and adds a learned covariance correction branch", section
"Hardware argument": the kernel keeps softmax's online maximum and rescale,
and runs two score branches over the same key / value tiles, a_j = scale q.k_j
and s_j = rho.k_j. Per query it accumulates, with p_j = exp(a_j - m) and m
the running maximum of the scores,

    l = sum_j p_j,  c = sum_j p_j s_j,  O1 = sum_j p_j v_j,  O2 = sum_j p_j s_j v_j,

and emits o = O1/l - (O2/l - (c/l)(O1/l)). The same section gives the
5-tuple (m, l, c, O1, O2) as the state that split-KV partials carry and merge.

Here those steps are taken in fp64 over consecutive key chunks, in key
order. A chunk's state joins the running state by rescaling both to the
larger maximum and adding, which is also how states of disjoint key sets
computed apart (split-KV decode, context parallelism) combine. The scores'
units are natural-log here (the kernels keep log2 units; that changes no
result).

Pinned by ``tests/test_oracle_stream_pins.py``: the row pins of the other two
forms (hand-derived examples, rho = 0 against SDPA, closed forms,
invariances), agreement with the explicit definition for every chunking and
every order of merging, and planted mistakes in the merge.
"""
from __future__ import annotations

import numpy as np

__all__ = ["chunk_state", "empty_state", "merge_states", "finish_state", "parallax_row_streamed"]


def empty_state(d_v):
    """The state of an empty key set: m = -inf, l = c = 0, O1 = O2 = 0."""
    return (-np.inf, 0.0, 0.0, np.zeros(d_v), np.zeros(d_v))


def chunk_state(q, rho, K, V, scale):
    """(m, l, c, O1, O2) of one query over one chunk of keys (news.chathome.org,
    "Hardware argument": the two branches share the chunk's maximum)."""
    if K.shape[0] == 0:
        return empty_state(V.shape[1])
    a = scale * (K @ q)
    s = K @ rho
    m = a.max()
    p = np.exp(a - m)
    return (m, p.sum(), (p * s).sum(), p @ V, (p * s) @ V)


def merge_states(x, y):
    """The state of the union of two disjoint key sets: both rescaled to the
    larger maximum, then added (the online rescale of the same section)."""
    m1, l1, c1, a1, b1 = x
    m2, l2, c2, a2, b2 = y
    m = max(m1, m2)
    if m == -np.inf:
        return x
    f1 = 0.0 if m1 == -np.inf else np.exp(m1 - m)
    f2 = 0.0 if m2 == -np.inf else np.exp(m2 - m)
    return (m, f1 * l1 + f2 * l2, f1 * c1 + f2 * c2, f1 * a1 + f2 * a2, f1 * b1 + f2 * b2)


def finish_state(st):
    """(o, lse) of a state: o = O1/l - (O2/l - (c/l)(O1/l)), lse = m + ln l.
    An empty key set gives o = 0, lse = -inf."""
    m, l, c, O1, O2 = st
    if l == 0.0:
        return np.zeros_like(O1), -np.inf
    o1 = O1 / l
    return o1 - (O2 / l - (c / l) * o1), m + np.log(l)


def parallax_row_streamed(q, rho, K, V, scale, chunk=None):
    """The streamed output of one query row over the keys in order, `chunk`
    keys at a time (None: all keys as one chunk)."""
    n = K.shape[0]
    step = n if not chunk else int(chunk)
    st = empty_state(V.shape[1])
    for j0 in range(0, n, max(step, 1)):
        st = merge_states(st, chunk_state(q, rho, K[j0:j0 + step], V[j0:j0 + step], scale))
    return finish_state(st)
