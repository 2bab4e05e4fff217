"""Comparison helpers shared by the GPU parity tests, the smoke check and the bench.

Tolerances (derived from the arithmetic; the bar for outputs also holds the
normwise 2e-3 relative error the decode step is specified to):
  * outputs: the kernel computes o (and y) in fp32 and rounds once to bf16
    (round to nearest even), so |out - ref| <= 1 bf16 ulp of |ref| (half an
    ulp for the rounding, the rest covers a binade crossing and fp32
    rounding), plus ATOL_OUT for outputs so close to zero that fp32
    accumulation error over K terms (~1e-7 absolute here) exceeds their ulp,
    plus RTOL_OUT for the fp32 error of the norm/gate (rsqrt, exp, division);
    normwise ||out - ref|| / ||ref|| <= 2e-3;
  * state: fp32 decay, correction and rank-1 write carry a few ulp (~1e-7
    relative) per token, so ||S - ref|| / ||ref|| <= 1e-5 and
    max|S - ref| <= 1e-5 max|ref|;
  * slots: every slot not named by an active row is bit-identical.
"""
from __future__ import annotations

import numpy as np

ATOL_OUT = 1e-6
RTOL_OUT = 1e-5
NORMWISE_OUT = 2e-3
STATE_REL = 1e-5


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits; subnormal floor)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_out(got, ref, what="out"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + ATOL_OUT + RTOL_OUT * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} elements exceed 1 bf16 ulp; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r} bound {bound[i]!r}")
    nref = np.linalg.norm(ref)
    if nref > 0:
        rel = np.linalg.norm(got - ref) / nref
        assert rel <= NORMWISE_OUT, f"{what}: normwise relative error {rel:.3e} > {NORMWISE_OUT}"


def check_state(got, ref, what="state"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    nref = np.linalg.norm(ref)
    if nref == 0:
        assert np.all(got == 0)
        return
    rel = np.linalg.norm(got - ref) / nref
    mx = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert rel <= STATE_REL, f"{what}: normwise relative error {rel:.3e} > {STATE_REL}"
    assert mx <= STATE_REL, f"{what}: max abs error / max|ref| = {mx:.3e} > {STATE_REL}"


def check_state_bf16(got, ref, what="bf16 state"):
    """A bf16 pool: the kernel rounds its fp32 state once, the oracle rounds its
    fp64 state once, so each element agrees to one bf16 ulp (fp32 error can
    move a value across a rounding boundary), plus 1e-6 max|ref| for values so
    small that fp32 cancellation error exceeds their ulp."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + 1e-6 * np.max(np.abs(ref))
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} elements off by more than 1 bf16 ulp; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r}")
    assert np.mean(got != ref) < 0.01, f"{what}: more than 1% of elements differ from the oracle"
