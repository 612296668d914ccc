import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-tie report of every GPU routing comparison (tokens whose fp64 k-th / (k+1)-th
    logit gap, or a gap inside the top k, is below 1e-4; and how many of them the GPU
    selected or ordered differently)."""
    try:
        from parity_util import NEAR_TIE_REPORTS
    except Exception:
        return
    if not NEAR_TIE_REPORTS:
        return
    tr = terminalreporter
    tr.write_sep("-", "near-tie report (routing parity)")
    tot = dict(T=0, near_set=0, near_order=0, mismatched=0, set_changed=0)
    for r in NEAR_TIE_REPORTS:
        tr.write_line("%s T=%d E=%d k=%d near_set=%d near_order=%d mismatched=%d set_changed=%d"
                      % (r["test"], r["T"], r["E"], r["k"], r["near_set"], r["near_order"],
                         r["mismatched"], r["set_changed"]))
        for key in tot:
            tot[key] += r[key]
    tr.write_line("total over %d comparisons: tokens=%d near_set=%d near_order=%d mismatched=%d "
                  "set_changed=%d" % (len(NEAR_TIE_REPORTS), tot["T"], tot["near_set"],
                                      tot["near_order"], tot["mismatched"], tot["set_changed"]))
