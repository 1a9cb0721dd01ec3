import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def load_golden(name):
    """Parse a ``key = values`` fixture under tests/golden/ into float lists."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split("=", 1)
            out[key.strip()] = [float(x) for x in val.split()]
    return out


def pytest_terminal_summary(terminalreporter):
    """Print the errors the parity tests measured (whole tensor, worst 64-token
    block of a head, worst sequence, final state, worst single state)."""
    try:
        import parity
    except ImportError:
        return
    if not parity.RECORDS:
        return
    tr = terminalreporter
    tr.section("parity errors (relative L2 against the fp64 oracle)")
    tr.write_line(f"{'case':64s} {'o':>9s} {'o block':>9s} {'o seq':>9s} {'state':>9s} "
                  f"{'st worst':>9s} {'bound':>7s}")
    for label, eo, eb, esq, es, esx, tol in parity.RECORDS:
        tr.write_line(f"{label[:64]:64s} {eo:9.2e} {eb:9.2e} {esq:9.2e} {es:9.2e} {esx:9.2e} "
                      f"{tol:7.0e}")
