import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """The closest calls of the GPU parity comparisons: worst error / bound
    per compared output under the plain bound (abs + rel*|want|), and under
    the bound actually applied where the two differ (stage-separated
    backward outputs with the fp32 noise allowance; end-to-end outputs with
    the wider relative scale)."""
    gu = sys.modules.get("gpu_util")
    if gu is None or not gu.RATIOS:
        return
    rows = gu.RATIOS
    tr = terminalreporter
    tr.section("parity: worst error / bound")
    tr.write_line(f"{len(rows)} comparisons; the 25 closest under the plain bound:")
    for what, plain, applied, kind in sorted(rows, key=lambda r: -r[1])[:25]:
        extra = "" if kind == "plain" else f"   ({kind} bound: {applied:.3g})"
        tr.write_line(f"  {plain:10.3g}  {what}{extra}")
    for kind, label in (("noise", "stage-separated with the fp32 noise allowance"),
                        ("scale", "end to end with the wider scale")):
        sel = [r for r in rows if r[3] == kind]
        over = [r for r in sel if r[1] > 1.0]
        worst = max((r[2] for r in sel), default=0.0)
        tr.write_line(f"{len(sel)} comparisons {label}: {len(over)} exceed the plain bound; "
                      f"worst ratio under the applied bound {worst:.3g}")
    plain = [r for r in rows if r[3] == "plain"]
    tr.write_line(f"{len(plain)} comparisons under the plain bound alone; worst "
                  f"{max((r[1] for r in plain), default=0.0):.3g}")
