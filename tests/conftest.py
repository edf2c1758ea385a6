import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)



def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    # the parity summaries tests.parity.Case.check_all collected in this session
    mod = sys.modules.get("tests.parity")
    PARITY_REPORT = getattr(mod, "PARITY_REPORT", None)
    if not PARITY_REPORT:
        return
    tr = terminalreporter
    tr.section("parity cases (excluded = near ties + fp32-explained id mismatches)")
    tr.write_line(f"{'case':64s} {'tok':>6s} {'rows':>7s} {'excl':>4s} {'tie':>3s} {'expl':>4s} "
                  f"{'reord':>5s} {'err/rms':>9s} {'ulp':>4s} {'flip':>5s}")
    for name, s in PARITY_REPORT:
        tr.write_line(f"{name[-64:]:64s} {s['tokens']:6d} {s['rows']:7d} {s['excluded']:4d} {s['near_tie']:3d} "
                      f"{s['explained']:4d} {s['reordered']:5d} {s['out_err_over_rms']:9.2e} {s['ulp']:4d} "
                      f"{s['flip_elems']:5d}")


@pytest.fixture(scope="session")
def repo_root():
    return ROOT
