"""Output tolerance used by every parity test (and by the mutant test that
shows the tolerance is tight enough to catch low-precision sum(x)).

Rule, per output element, with y_ref the oracle's fp64 value and
absdot = sum_k |x[m,k] * w_hat[n,k]| (also from the oracle):
  * f16 / bf16 outputs pass when |y - y_ref| <= 1 ulp of the dtype at y_ref,
    or, where the fp32 sum cancels, |y - y_ref| <= 1e-5 * absdot;
  * f32 outputs pass when |y - y_ref| <= 1e-5 * absdot.
The 1-ulp bound is the workload's stated bar (the MLX pull request checks half
a bf16 step of a float64 reference); 1e-5 * sum|x*w| is the f32 bar, used as the
floor for cancelling sums where the ulp of the result is far below the fp32
rounding of its terms.  How often the second clause was needed is reported.
"""
from __future__ import annotations

import numpy as np

_PREC = {"bf16": (8, -126), "f16": (11, -14), "f32": (24, -126)}
REL_FLOOR = 1e-5


def ulp(v: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of ``dtype`` at |v| (the subnormal spacing below the normal range)."""
    p, emin = _PREC[dtype]
    a = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(a > 0, np.maximum(e, emin), emin)
    return np.ldexp(1.0, (e - (p - 1)).astype(np.int64))


def check(y, y_ref, absdot, dtype):
    """Return (ok_mask, n_needed_floor) comparing GPU outputs y (float64 values
    of the dtype) to the oracle.  Non-finite reference values must match
    exactly (same inf / NaN)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    absdot = np.asarray(absdot, dtype=np.float64)
    fin = np.isfinite(y_ref) & np.isfinite(absdot)
    err = np.abs(y - y_ref)
    floor_ok = err <= REL_FLOOR * absdot
    if dtype == "f32":
        ok = floor_ok
        needed = 0
    else:
        ulp_ok = err <= ulp(y_ref, dtype)
        ok = ulp_ok | floor_ok
        needed = int(np.count_nonzero(fin & ~ulp_ok & floor_ok))
    same_nonfinite = (np.isnan(y) & np.isnan(y_ref)) | (y == y_ref)
    ok = np.where(fin, ok, same_nonfinite)
    return ok, needed


def assert_close(y, y_ref, absdot, dtype, what=""):
    ok, needed = check(y, y_ref, absdot, dtype)
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(
            f"{what}: {len(bad)} / {ok.size} outputs out of tolerance; first at {i}: "
            f"y={np.asarray(y)[i]!r} ref={np.asarray(y_ref)[i]!r} absdot={np.asarray(absdot)[i]!r}")
    return needed
