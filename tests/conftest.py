"""Shared pytest setup: the repository root on sys.path and the `gpu` marker."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Achieved attention errors against the float64 oracle: one line per
    whole-output comparison (the full-size workloads), then the worst of the
    sampled comparisons, so the margin to the tolerances is on record.  "beyond
    rounding" is the largest |gpu - exact| minus half an ulp of the output dtype
    at the exact value, the quantity bounded by the max-abs tolerance."""
    helpers = sys.modules.get("gpu_helpers")
    log = getattr(helpers, "ERROR_LOG", None)
    if not log:
        return
    tr = terminalreporter
    tr.write_sep("-", "attention errors against the float64 oracle "
                      f"(bounds: max-abs {helpers.MAX_ABS:g} beyond the output's rounding, "
                      f"rel-L2 {helpers.REL_L2:g}, lse {helpers.LSE_MAX_ABS:g})")
    sampled = [e for e in log if e[5] is None]
    if sampled:
        worst_abs = max(sampled, key=lambda e: e[1])
        worst_ex = max(sampled, key=lambda e: e[6])
        worst_rel = max(sampled, key=lambda e: e[2])
        tr.write_line(f"{len(sampled)} sampled comparisons: worst max-abs {worst_abs[1]:.3e} "
                      f"({worst_abs[0]}), worst beyond rounding {worst_ex[6]:.3e} "
                      f"({worst_ex[0]}), worst rel-L2 {worst_rel[2]:.3e} ({worst_rel[0]})")
    for what, max_abs, rel, lse_err, rows, total, excess in log:
        if total is None:
            continue
        lse_s = "-" if lse_err is None else f"{lse_err:.3e}"
        tr.write_line(f"{what}: {rows} of {total} rows, max-abs {max_abs:.3e} "
                      f"(beyond rounding {excess:.3e}), rel-L2 {rel:.3e}, lse max-abs {lse_s}")
