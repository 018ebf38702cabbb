import os
import sys
from collections import OrderedDict

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU check")


@pytest.fixture(autouse=True)
def _name_selection_checks(request):
    """Selection checks record the test they ran in."""
    import helpers
    helpers.set_current_test(request.node.nodeid)
    yield


def pytest_terminal_summary(terminalreporter):
    """Per test: the selection checks' largest undecided share of K, smallest
    overlap with the oracle's sets and most differing picks; and the largest
    logit error seen, relative to sum |q k| / sqrt(D)."""
    import helpers
    rec = helpers.SELECTION_RECORD
    if not rec and not helpers.LOGIT_RECORD and not helpers.LSE_RECORD:
        return
    tr = terminalreporter
    tr.section("selection parity")
    agg = OrderedDict()
    for test, _what, _h, K, und, ov, diff in rec:
        a = agg.setdefault(test, {"checks": 0, "K": set(), "und": 0, "share": 0.0, "ov": 1.0, "diff": 0,
                                  "sum": 0.0})
        a["checks"] += 1
        a["sum"] += und / K
        a["K"].add(K)
        a["und"] = max(a["und"], und)
        a["share"] = max(a["share"], und / K)
        a["ov"] = min(a["ov"], ov)
        a["diff"] = max(a["diff"], diff)
    for test, a in agg.items():
        ks = sorted(a["K"])
        tr.write_line(f"{test}: {a['checks']} head checks, K {ks[0]}..{ks[-1]}, max undecided {a['und']} "
                      f"({100 * a['share']:.3f} % of K; mean {100 * a['sum'] / a['checks']:.3f} %), min overlap {a['ov']:.6f}, max differing picks {a['diff']}")
    if rec:
        tr.write_line(f"all: {len(rec)} head checks, max undecided share "
                      f"{100 * max(r[4] / r[3] for r in rec):.3f} % (mean {100 * sum(r[4] / r[3] for r in rec) / len(rec):.3f} %), "
                      f"min overlap {min(r[5] for r in rec):.6f}")
    if helpers.LOGIT_RECORD:
        tr.write_line(f"logit error: at most {max(helpers.LOGIT_RECORD):.3e} x sum|q k|/sqrt(D) "
                      f"(bound {helpers.C_Z:.3e})")
    if helpers.LSE_RECORD:
        tr.write_line(f"candidate lse error: at most {max(helpers.LSE_RECORD):.3f} of its bound")
