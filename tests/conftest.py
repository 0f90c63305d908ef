import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running oracle work (minutes)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Worst logit error of every GPU parity case that ran, against the bounds
    (max-abs 5e-2, rel-L2 1e-2), so the headroom is on record even under -q."""
    from tests import _harness

    if not _harness.PARITY_RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity headroom (worst over steps and lanes)")
    tr.write_line(f"{'case':48s} {'max-abs':>9s} {'rel-L2':>9s} {'steps':>6s} {'ids':>5s}")
    for case, ma, rl, steps, ids in _harness.PARITY_RECORDS:
        tr.write_line(f"{case:48s} {ma:9.3e} {rl:9.3e} {steps:6d} {ids:5d}")
