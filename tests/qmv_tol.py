"""Output tolerance used by every parity test (and by the mutant test that
shows the tolerance is tight enough to catch low-precision sum(x)).

Rule, per output element, with y_ref the oracle's fp64 value and
absdot = sum_k |x[m,k] * w_hat[n,k]| (also from the oracle):
  * f16 / bf16 outputs pass when |y - y_ref| <= 1 ulp of the dtype at y_ref,
    or, where the fp32 sum cancels, |y - y_ref| <= REL_FLOOR * absdot;
  * f32 outputs pass when |y - y_ref| <= REL_FLOOR * absdot.

Where the floor comes from.  The workload states two bars: 1 ulp for f16 /
bf16 outputs, and 1e-5 * sum|x*w| for f32 outputs.  A f16 / bf16 output is the
round-to-nearest of the kernel's fp32 accumulator, and that accumulator is held
to the f32 bar.  Where the result cancels (|y_ref| far below absdot) its ulp in
the output dtype falls below what any fp32 accumulation of absdot-sized terms
can resolve, and only the f32 bar is meaningful; the floor clause is exactly
that bar.  It can only decide an element whose ulp is below REL_FLOOR * absdot
(otherwise the ulp clause is the looser one), so every use of it is in a
cancelling output.

How often the floor decided an output is counted per comparison (``needed``):
assert_close fails when more than ``max_floor_frac`` of the finite outputs (plus
one) needed it, and every comparison is recorded in RECORDS (what, outputs,
needed, and the worst err / absdot among them) for the session summary that
tests/conftest.py prints.
"""
from __future__ import annotations

import numpy as np

_PREC = {"bf16": (8, -126), "f16": (11, -14), "f32": (24, -126)}
REL_FLOOR = 1e-5
# default bound on the share of outputs the floor may decide (N(0,1) x: a few
# per thousand cancel that far); precision cases pass their own
FLOOR_FRAC = 0.02
RECORDS: list[dict] = []


def ulp(v: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of ``dtype`` at |v| (the subnormal spacing below the normal range)."""
    p, emin = _PREC[dtype]
    a = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(a > 0, np.maximum(e, emin), emin)
    return np.ldexp(1.0, (e - (p - 1)).astype(np.int64))


def check_stats(y, y_ref, absdot, dtype):
    """Return (ok_mask, n_needed_floor, worst, n_finite): ``worst`` is the
    largest err / absdot among the outputs the floor decided (0 if none)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    absdot = np.asarray(absdot, dtype=np.float64)
    fin = np.isfinite(y_ref) & np.isfinite(absdot)
    err = np.abs(y - y_ref)
    floor_ok = err <= REL_FLOOR * absdot
    worst = 0.0
    if dtype == "f32":
        ok = floor_ok
        needed = 0
        # f32 outputs are all held to the floor: record their worst ratio
        sel = fin & (absdot > 0)
        if sel.any():
            worst = float(np.max(err[sel] / absdot[sel]))
    else:
        ulp_ok = err <= ulp(y_ref, dtype)
        ok = ulp_ok | floor_ok
        used = fin & ~ulp_ok & floor_ok
        needed = int(np.count_nonzero(used))
        if needed:
            with np.errstate(divide="ignore", invalid="ignore"):
                worst = float(np.max(err[used] / absdot[used]))
    same_nonfinite = (np.isnan(y) & np.isnan(y_ref)) | (y == y_ref)
    ok = np.where(fin, ok, same_nonfinite)
    return ok, needed, worst, int(np.count_nonzero(fin))


def check(y, y_ref, absdot, dtype):
    """Return (ok_mask, n_needed_floor)."""
    ok, needed, _, _ = check_stats(y, y_ref, absdot, dtype)
    return ok, needed


def assert_close(y, y_ref, absdot, dtype, what="", max_floor_frac=FLOOR_FRAC):
    ok, needed, worst, nfin = check_stats(y, y_ref, absdot, dtype)
    # worst: err / absdot among the outputs the floor decided (f16 / bf16) or
    # among all outputs (f32, where the floor is the whole bar)
    RECORDS.append({"what": what, "dtype": dtype, "outputs": int(ok.size), "needed": needed, "worst": worst})
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(
            f"{what}: {len(bad)} / {ok.size} outputs out of tolerance; first at {i}: "
            f"y={np.asarray(y)[i]!r} ref={np.asarray(y_ref)[i]!r} absdot={np.asarray(absdot)[i]!r}")
    if needed > max_floor_frac * nfin + 1:
        raise AssertionError(f"{what}: the fp32 floor decided {needed} of {nfin} outputs "
                             f"(bound {max_floor_frac:.3f}); worst err/absdot {worst:.3g}")
    return needed
