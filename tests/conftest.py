import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library, loaded through the package binding."""
    import gated_delta_rule_112_b200 as gdn
    return gdn


@pytest.fixture(autouse=True)
def _parity_record_owner(request):
    """Tags every parity comparison with the test that makes it."""
    from tests import parity
    parity.CURRENT_TEST["id"] = request.node.nodeid
    yield
    parity.CURRENT_TEST["id"] = None


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Parity margins: relative L2 and max-abs of every full-size workload
    comparison (the tests named test_workload_*), and the worst relative L2
    over all comparisons; all records go to $GDN_PARITY_MARGINS as JSON."""
    from tests import parity
    recs = parity.RECORDS
    if not recs:
        return
    path = os.environ.get("GDN_PARITY_MARGINS")
    if path:
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump(recs, f, indent=1)
    tr = terminalreporter
    tr.section("parity margins (rel-L2 / max-abs against the fp64 oracle)")
    for r in recs:
        if "test_workload" in (r["test"] or ""):
            name = r["test"].split("::")[-1]
            tr.write_line(f"{name:48s} {r['tensor']:28s} rel-L2 {r['rel_l2']:.3e} "
                          f"(tol {r['tol']:.0e})  max-abs {r['max_abs']:.3e}")
    worst = max(recs, key=lambda r: r["rel_l2"] / r["tol"])
    tr.write_line(f"{len(recs)} comparisons; closest to its tolerance: "
                  f"{worst['test'].split('::')[-1]} {worst['tensor']} rel-L2 "
                  f"{worst['rel_l2']:.3e} of {worst['tol']:.0e}")
