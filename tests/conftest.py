import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The measured errors of every GPU parity check (also on -q runs)."""
    try:
        from gpu_helpers import RECORDS
    except Exception:
        return
    if not RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", "measured parity errors (max over checked tokens)")
    for r in RECORDS:
        tr.write_line(f"{r['check']:<44} tokens {r['tokens']:>5}  h {r['h_rel_err']:.1e}  "
                      f"chain {r['chain_rel_err']:.1e}  e2e(clean) {r['e2e_rel_err_clean']:.1e}  "
                      f"e2e(all) {r['e2e_rel_err_all']:.1e}  elementwise {r['elementwise_clean']:.1e}  "
                      f"flip tokens {r['flip_tokens']}")
