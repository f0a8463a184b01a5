import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def lib():
    """The compiled C-ABI library through its Python binding (GPU tests only)."""
    import activation_quantization_b200 as aq
    return aq


def pytest_terminal_summary(terminalreporter):
    """Boundary-window counts of the parity comparisons that ran (GPU tests).

    ``in_window``: elements whose oracle pre-rounding value lies within the 1e-6
    window of a rounding boundary; ``exempt``: those of them whose GPU code differs
    (the mismatches the window excuses, bounded by 1e-4 of the elements);
    ``scale_exempt``: block scales that differ inside their window.
    """
    parity = sys.modules.get("tests.parity")
    log = getattr(parity, "WINDOW_LOG", None)
    if not log:
        return
    import json
    tr = terminalreporter
    tr.section("boundary-window counts (transform + quantise parity)")
    totals = {}
    for e in log:
        t = totals.setdefault(e["fmt"], dict(elements=0, in_window=0, exempt=0, blocks=0, scale_in_window=0,
                                             scale_exempt=0, comparisons=0))
        for k in ("elements", "in_window", "exempt", "blocks", "scale_in_window", "scale_exempt"):
            t[k] += e[k]
        t["comparisons"] += 1
    for fmt, t in sorted(totals.items()):
        tr.write_line(f"{fmt:6s} {t['comparisons']:4d} comparisons, {t['elements']:12d} elements: "
                      f"in window {t['in_window'] / t['elements']:.3e}, excused mismatches "
                      f"{t['exempt'] / t['elements']:.3e} ({t['exempt']}), scales in window "
                      f"{t['scale_in_window'] / t['blocks']:.3e}, excused scale mismatches {t['scale_exempt']}")
    big = sorted(log, key=lambda e: -e["elements"])[:12]
    for e in big:
        tr.write_line(f"  {e['test']}: {e['fmt']} {e['rows']}x{e['d_in']}: in window {e['in_window']}, "
                      f"excused {e['exempt']}, scale excused {e['scale_exempt']}")
    path = os.environ.get("WUSH_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump({"per_format": totals, "comparisons": log}, f, indent=1)
