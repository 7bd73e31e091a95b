import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running oracle case")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Errors of every parity comparison of the session, one line each."""
    import parity_log
    if not parity_log.RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity against the oracle ({len(parity_log.RECORDS)} comparisons)")
    for what, dtype, ma, rl, tma, trl in parity_log.RECORDS:
        tr.write_line(f"{what:<48} {dtype:<5} max_abs {ma:.3e} / {tma:g}   "
                      f"rel_l2 {rl:.3e} / {trl:g}   margin {min(tma - ma, trl - rl) >= 0}")
