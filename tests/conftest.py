import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(ROOT)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload checks")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Counts of the elementwise float comparisons with the oracle: how many
    elements lay beyond the strict bound |gpu - ref| <= 1e-2 + 1e-2 |ref|, per
    check that had any (helpers.PARITY)."""
    helpers = sys.modules.get("helpers")
    recs = getattr(helpers, "PARITY", None)
    if not recs:
        return
    tr = terminalreporter
    n_el = sum(r["elements"] for r in recs)
    n_bad = sum(r["beyond_strict"] for r in recs)
    tr.write_sep("-", "parity: |gpu - ref| <= 1e-2 + 1e-2 |ref| elementwise")
    tr.write_line(f"{len(recs)} float comparisons, {n_el} elements, {n_bad} beyond the strict bound")
    for r in recs:
        if r["beyond_strict"]:
            tr.write_line(f"  {r['what']}: {r['beyond_strict']} of {r['elements']} within the "
                          f"{r['allowance']} allowance (worst err/tol {r['worst_err_over_tol']:.3g})")
    path = os.environ.get("MOE_PARITY_LOG")
    if path:
        with open(path, "w") as f:
            json.dump(recs, f, indent=1)


@pytest.fixture(autouse=True)
def _library_kernel_choice():
    """Every test starts and ends with the library choosing its kernels by
    shape (a test may force variants with helpers.force_kernels)."""
    yield
    helpers = sys.modules.get("helpers")
    if helpers is not None:
        helpers.reset_kernels()
