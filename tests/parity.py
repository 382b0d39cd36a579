"""Shared comparison rule for GPU-vs-oracle parity tests.

Floating-point outputs (bf16 Out, dQ, dK, dV) must be within 1e-2 max-abs and 1e-2 relative L2 of
the fp64 oracle.  Where a reference value is so large that 1e-2 is below bf16 resolution
(|x| > 2.56, where one bf16 ulp exceeds 1e-2), an element also passes within one bf16 ulp of the
reference.  The relative-L2 denominator is floored at 1e-2 * sqrt(n): a reference that is exactly
zero (a token that sees only its own key has dQ = 0 in closed form) then needs an RMS error of at
most 1e-4 instead of a ratio over zero.  LSE (fp32) must be within 1e-3 max-abs.
"""
import numpy as np
import torch

ATOL, RTOL_L2, LSE_ATOL = 1e-2, 1e-2, 1e-3


def bf16_ulp(x):
    ax = np.maximum(np.abs(x), 1e-30)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def check_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    tol = np.maximum(ATOL, bf16_ulp(ref))
    bad = err > tol
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), ATOL * np.sqrt(ref.size))
    assert not bad.any() and rel <= RTOL_L2, (
        f"{what}: {bad.sum()} elements over tolerance, max abs {err.max():.3e}, rel L2 {rel:.3e}")
    return float(err.max()), float(rel)


def check_lse(got, ref, what="lse"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fin = np.isfinite(ref)
    assert np.all(np.isneginf(got[~fin])), f"{what}: rows without keys must be -inf"
    err = np.abs(got[fin] - ref[fin])
    assert err.size == 0 or err.max() <= LSE_ATOL, f"{what}: max abs {err.max():.3e}"


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()
