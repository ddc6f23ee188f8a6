import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session", autouse=True)
def _build_oracle():
    import oracle
    oracle.build()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One line per GPU parity case (tests.parity.REPORT, filled by tests.gpu_util.run_case):
    the clean / unclean token counts of the routing comparison, the tokens whose decision
    differs from the oracle's (inside the 1e-3 margin), and the y errors."""
    from tests.parity import REPORT as PARITY_REPORT
    if not PARITY_REPORT:
        return
    tr = terminalreporter
    tr.section("parity report (GPU vs fp64 oracle)")
    tr.write_line("case | tokens | clean | unclean | differing | y tokens | max|err| | rel-L2 | "
                  "max|err| vs oracle decision | rel-L2 vs oracle decision")
    for r in PARITY_REPORT:
        tr.write_line(f"{r['case']} | {r['T']} | {r['clean']} | {r['unclean']} | {r['differing']} | "
                      f"{r['y_tokens']} | {r['max_abs']:.3e} | {r['rel_l2']:.3e} | "
                      f"{r['max_abs_own']:.3e} | {r['rel_l2_own']:.3e}")
