"""Shared tolerances and comparison for the GPU-vs-oracle parity tests.

Tolerances for bf16 inputs with fp32 accumulation: max |out - ref| <= 2e-2,
relative L2 ||out - ref|| / ||ref|| <= 5e-3 over the compared values, and
|lse - ref| <= 1e-3 (where lse is finite; -inf must match exactly).
The gradient bounds are below.
"""
import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3

# Gradients (the backward pass), per tensor: max |g - ref| <= GRAD_MAX_REL *
# max(1, max|ref|) and ||g - ref|| / ||ref|| <= GRAD_REL_L2.  The pages fix no
# gradient tolerance; test_grad_tolerance_cpu.py derives these from a CPU model
# of the kernels' bf16 operand rounding and checks the headroom they leave.
GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


def to_np(t):
    if hasattr(t, "detach"):
        t = t.detach().float().cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def assert_close(out, ref, lse=None, ref_lse=None, what="", scale_abs=False):
    """scale_abs: for stress inputs whose outputs exceed O(1), the max-abs bound
    is 2e-2 * max(1, max|ref|): the output is stored in bf16 (8 significant
    bits), so its rounding alone is ~2^-9 |ref| and operand rounding of p and
    p*s grows with the output scale as well."""
    out, ref = to_np(out), to_np(ref)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref)
    max_abs = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(out - ref)) / den if den > 0 else float(np.linalg.norm(out - ref))
    bound = MAX_ABS * max(1.0, float(np.abs(ref).max())) if scale_abs else MAX_ABS
    assert max_abs <= bound, f"{what}: max abs err {max_abs:.3e} > {bound:.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e} > {REL_L2}"
    if lse is not None:
        lse, ref_lse = to_np(lse), to_np(ref_lse)
        fin = np.isfinite(ref_lse)
        assert (np.isneginf(lse) == np.isneginf(ref_lse)).all(), f"{what}: -inf lse mismatch"
        if fin.any():
            lerr = float(np.abs(lse[fin] - ref_lse[fin]).max())
            assert lerr <= LSE_ABS, f"{what}: lse err {lerr:.3e} > {LSE_ABS}"
    return max_abs, rel
