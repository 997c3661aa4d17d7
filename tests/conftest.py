"""Shared pytest configuration: the ``gpu`` marker is registered in pytest.ini.

GPU tests fail loudly (never skip) when CUDA or the compiled library is
missing, so a GPU run can never pass on a fallback path.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Totals of the output comparisons: how many outputs were compared, how
    many the fp32 floor clause decided, and the worst err / sum|x*w| among
    those.  With QMV_TOL_REPORT set, every comparison is also written there as
    JSON."""
    try:
        import qmv_tol
    except ImportError:
        return
    recs = qmv_tol.RECORDS
    if not recs:
        return
    total = sum(r["outputs"] for r in recs)
    needed = sum(r["needed"] for r in recs)
    worst = max(r["worst"] for r in recs)
    terminalreporter.write_line(
        f"tolerance: {len(recs)} comparisons, {total} outputs, floor clause decided {needed} "
        f"({needed / max(total, 1):.2e}), worst err/sum|x*w| there {worst:.3g} (floor {qmv_tol.REL_FLOOR:g})")
    path = os.environ.get("QMV_TOL_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(recs, f)
