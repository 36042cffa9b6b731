"""Where the gradient tolerance comes from (CPU, no GPU needed).

The pages give the forward only (gist.science, "Technical overview:
Parallax ...", "Method: Parallax / Core mechanism"), so the gradient bounds
GRAD_REL_L2 and GRAD_MAX_REL (parity.py) are not fixed by them.  This test
derives the error that the backward kernels' arithmetic is expected to show,
by replaying their rounding on the CPU, and asserts that the bounds leave
headroom above it without being loose enough to pass a wrong gradient.

The rounding model follows what the kernels store and feed to the tensor
cores, in the notation of the gradient oracle (oracle/plx_oracle_bwd.py):

- the training forward's out and o_bar are bf16 (so g_bar = dO . o_bar and
  D = dO . out + s_bar g_bar see bf16 values);
- the MMA operands W_hat, scale*dA and dS are rounded to bf16 (q, k, v, rho
  and dO are bf16 inputs already), accumulated in fp64 here (fp32 on the
  device: far below the bf16 operand error);
- dq, dk, dv, dr are stored as bf16.

Everything else (scores, softmax weights, g, g_bar, D) is exact here.  The
workloads are those of the GPU gradient tests (test_bwd_gpu.py).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import plx_oracle_bwd as ob
from parity import GRAD_MAX_REL, GRAD_REL_L2
from parameterized_local_linear_plx_b200 import inputs

# the bounds must sit at least this far above the modelled error
HEADROOM = 2.5


def bf16(x):
    """Round an fp64 array to bf16 (round to nearest even) and back."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).bfloat16().double().numpy()


def modelled_block(Q, R, K, V, dO, out, obar, mask, scale, drop_sbar=False):
    """Gradients of one (b, query head) block with the kernels' rounding."""
    W = ob._softmax_masked(scale * (Q @ K.T), mask)
    S = R @ K.T
    G = dO @ V.T
    sbar = (W * S).sum(1, keepdims=True)
    gbar = (dO * obar).sum(1, keepdims=True)
    D = (dO * out).sum(1, keepdims=True) + sbar * gbar
    sb = 0.0 if drop_sbar else sbar
    w_hat = bf16(W * (1 - S + sb))
    dS = bf16(W * (gbar - G))
    dA = bf16(scale * W * (G * (1 - S + sb) + S * gbar - D))
    return dA @ K, dA.T @ Q + dS.T @ R, w_hat.T @ dO, dS @ K


def modelled_errors(B, Hq, Hkv, N, d, seed, r_scale=0.1, q_mult=1.0, drop_sbar=False):
    """Per gradient (dq, dk, dv, dr): (rel L2, max abs / max(1, max|ref|))
    between the rounding model and the exact fp64 gradient."""
    q, k, v, r = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=seed, r_scale=r_scale)
    if q_mult != 1.0:
        q = (q.float() * q_mult).bfloat16()
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(seed + 7)).bfloat16()
    qn, kn, vn, rn, don = (t.double().numpy() for t in (q, k, v, r, do))
    exact = oracle.prefill_backward_closed(qn, kn, vn, rn, don, True)
    out, _ = oracle.prefill_effective(qn, kn, vn, rn, True)
    obar, _ = oracle.prefill_aux(qn, kn, vn, rn, True)
    out, obar = bf16(out), bf16(obar)
    mask = ob._mask(N, True)
    scale = 1.0 / np.sqrt(d)
    G = Hq // Hkv
    model = [np.zeros_like(x) for x in exact]
    for b in range(B):
        for h in range(Hq):
            gq, gk, gv, gr = modelled_block(qn[b, h], rn[b, h], kn[b, h // G], vn[b, h // G], don[b, h],
                                            out[b, h], obar[b, h], mask, scale, drop_sbar)
            model[0][b, h] += gq
            model[3][b, h] += gr
            model[1][b, h // G] += gk
            model[2][b, h // G] += gv
    res = []
    for x, y in zip(model, exact):
        x = bf16(x)
        rel = float(np.linalg.norm(x - y) / np.linalg.norm(y))
        mx = float(np.abs(x - y).max() / max(1.0, np.abs(y).max()))
        res.append((rel, mx))
    return res


WORKLOADS = {
    "tiny B=1 H=1 N=256 d=64": dict(B=1, Hq=1, Hkv=1, N=256, d=64, seed=0),
    "GQA B=2 Hq=4 Hkv=2 N=333 d=128": dict(B=2, Hq=4, Hkv=2, N=333, d=128, seed=1),
    "GQA B=2 Hq=4 Hkv=2 N=333 d=64": dict(B=2, Hq=4, Hkv=2, N=333, d=64, seed=2),
    "stress q*4 rho~N(0,1) N=512 d=128": dict(B=1, Hq=2, Hkv=1, N=512, d=128, seed=3, r_scale=1.0, q_mult=4.0),
}


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_gradient_bounds_leave_headroom_over_bf16_rounding(name):
    for g, (rel, mx) in zip(("dq", "dk", "dv", "dr"), modelled_errors(**WORKLOADS[name])):
        assert rel * HEADROOM <= GRAD_REL_L2, f"{name} {g}: modelled rel L2 {rel:.2e}"
        assert mx * HEADROOM <= GRAD_MAX_REL, f"{name} {g}: modelled max {mx:.2e}"
        # the model is not trivially exact either: bf16 operands leave a trace
        assert rel > 1e-4, f"{name} {g}: modelled rel L2 {rel:.2e} implausibly small"


def test_gradient_bounds_reject_a_dropped_term():
    """A plausible kernel mistake, s_bar left out of w_hat and dA, must fail
    the relative bound on the stress workload (large probe)."""
    errs = modelled_errors(**WORKLOADS["stress q*4 rho~N(0,1) N=512 d=128"], drop_sbar=True)
    assert max(rel for rel, _ in errs) > GRAD_REL_L2
