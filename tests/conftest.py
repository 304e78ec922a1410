import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Prints the parity errors that the GPU tests measured, each beside its bound, and writes
    them as JSON when DPCLIP_PARITY_MARGINS names a file."""
    mod = sys.modules.get("tests.gpu_helpers")
    rows = getattr(mod, "MARGINS", None) if mod else None
    if not rows:
        return
    terminalreporter.write_sep("-", "parity errors measured against the oracle (value / bound)")
    worst = {}
    for test, item, quantity, value, bound in rows:
        key = (test, quantity)
        if key not in worst or value / bound > worst[key][1] / worst[key][2]:
            worst[key] = (item, value, bound)
    for (test, quantity), (item, value, bound) in sorted(worst.items()):
        terminalreporter.write_line(f"{test:52s} {quantity:6s} worst {value:10.3e} / {bound:8.1e} "
                                    f"({100.0 * value / bound:5.1f}% of bound) at {item}")
    out = os.environ.get("DPCLIP_PARITY_MARGINS")
    if out:
        import json

        with open(out, "w") as f:
            json.dump([{"test": t, "item": i, "quantity": q, "value": v, "bound": b} for t, i, q, v, b in rows],
                      f, indent=1)
