"""Checks of the fp32 training step against the fp64 oracle (shared by the GPU tests and the CPU
tests that show the checks have teeth).

Gradients: element by element, |got - oracle| <= 1e-5 (|oracle| + S2) + F (error_bound.py), and the
fp32 error budget (fp32_budget.py) on the quantiles and the maximum.

SGD updates: the stored parameters change by exactly the update, so the change is checked, not the
updated value (whose own magnitude would hide a wrong sign or rate):
  - against the kernel's own gradient, to fp32 rounding: the new value is the fp32 rounding of
    w - lr g (one or two roundings: with or without a fused multiply-add), so
    |(after - before) + lr g| <= 2^-23 (|lr g| + |after|);
  - against the oracle's gradient, with the gradient's tolerance scaled by lr, plus the same
    rounding allowance.
"""
from __future__ import annotations

import numpy as np

from error_bound import tolerance
from fp32_budget import check_within_budget

RTOL = 1e-5
U2 = 2.0 ** -23          # two fp32 roundings (product and difference), each at most 2^-24 relative


def check_grad(got, want, S2, F, what, rtol=RTOL):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    lim = tolerance(want, S2, F, rtol)
    err = np.abs(got - want)
    bad = ~(err <= lim)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err / (lim + 1e-300), -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} entries outside rtol (|o| + S2) + F; worst at {i}: "
                             f"got {got[i]!r} oracle {want[i]!r} bound {lim[i]:.3g}")


def check_grad_and_budget(got, want, S2, F, refs, what):
    check_grad(got, want, S2, F, what)
    check_within_budget(got, want, refs, what, allowance=F)


def check_update_own(before, after, g, lr, what):
    """after - before == -lr g to fp32 rounding (g: the kernel's own gradient, fp32)."""
    before, after, g = (np.asarray(a, np.float64) for a in (before, after, g))
    delta = after - before                       # exact: both are fp32 values of nearby magnitude
    step = lr * g
    err = np.abs(delta + step)
    lim = U2 * (np.abs(step) + np.abs(after))
    bad = ~(err <= lim)
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{bad.size} updates differ from -lr g beyond fp32 rounding; "
                           f"worst {float((err / (lim + 1e-300)).max()):.3g} x the allowance")


def check_update_oracle(before, after, g_oracle, S2, F, lr, what):
    """after - before against -lr g_oracle: the gradient's tolerance times lr, plus the update's rounding."""
    before, after, g_oracle = (np.asarray(a, np.float64) for a in (before, after, g_oracle))
    delta = after - before
    err = np.abs(delta + lr * g_oracle)
    lim = lr * tolerance(g_oracle, S2, F) + U2 * (lr * np.abs(g_oracle) + np.abs(after))
    bad = ~(err <= lim)
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{bad.size} updates differ from -lr g_oracle; worst "
                           f"{float((err / (lim + 1e-300)).max()):.3g} x the bound")


# ---- planted mistakes (applied to the oracle's expected values, never to the code under test)

def corrupt_column(g, col=None, factor=1.05):
    """One output column of a weight gradient [out][in] scaled by `factor` (5 % off by default)."""
    g = np.array(g, np.float64, copy=True)
    col = int(np.argmax(np.abs(g).sum(0))) if col is None else col
    g[:, col] *= factor
    return g


def corrupt_row(g, row, factor=1.05):
    g = np.array(g, np.float64, copy=True)
    g[row] *= factor
    return g
