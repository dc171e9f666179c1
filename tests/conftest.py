import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libdualqk.so")
    config.addinivalue_line("markers", "slow: large-size case")


@pytest.fixture(scope="session")
def oracle_mod():
    from oracle import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """The output-parity margins every GPU case measured (max abs error and
    max per-row relative error against the oracle), so a quiet run shows how
    far each case is from the 2e-3 / 1e-2 bounds."""
    import harness
    rec = harness.PARITY_RECORDS
    if not rec:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity margins ({len(rec)} output comparisons; bounds 2e-3 abs, 1e-2 row-relative)")
    worst_abs = max(rec, key=lambda r: r[1])
    worst_rel = max(rec, key=lambda r: r[2])
    tr.write_line(f"worst max-abs error {worst_abs[1]:.3e} in {worst_abs[0]}")
    tr.write_line(f"worst row-relative error {worst_rel[2]:.3e} in {worst_rel[0]}")
    per_test = {}
    for name, a, r in rec:
        pa, pr = per_test.get(name, (0.0, 0.0))
        per_test[name] = (max(pa, a), max(pr, r))
    for name, (a, r) in sorted(per_test.items()):
        tr.write_line(f"  {a:.3e} abs  {r:.3e} rel  {name}")
