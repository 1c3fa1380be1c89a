import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_terminal_summary(terminalreporter):
    """Counts of compared and near-tie decisions of the verifier parity tests."""
    try:
        from tests.parity import REPORTS
    except Exception:
        return
    if not REPORTS:
        return
    tr = terminalreporter
    tr.section("verifier parity: compared sequences and near ties")
    tot = [0, 0, 0, 0]
    for name, r in REPORTS:
        tr.write_line(f"{name}: {r.rows} sequences, {r.compared} compared, "
                      f"{r.accept_ties} accept ties, {r.draw_ties} draw ties, {r.invalid} invalid")
        for k, v in enumerate((r.rows, r.compared, r.accept_ties, r.draw_ties)):
            tot[k] += v
    tr.write_line(f"all: {tot[0]} sequences, {tot[1]} compared "
                  f"({100.0 * tot[1] / max(1, tot[0] - 0):.1f}%), {tot[2]} accept ties, "
                  f"{tot[3]} draw ties")
