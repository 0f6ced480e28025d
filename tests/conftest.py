import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Per test: codes compared, mismatched, excused by the boundary rule
    (|c_gpu - c_orc| = 1 within 1e-5 relative of the decision boundary) and
    the excused fraction; also written as JSON to $KVQ_PARITY_REPORT if set."""
    import json
    import sys as _sys
    par = _sys.modules.get("parity")
    if par is None or not par.REPORTS:
        return
    agg = {}
    for tid, r in par.REPORTS:
        a = agg.setdefault(tid, [0, 0, 0, 0])
        a[0] += r.n
        a[1] += r.mismatched
        a[2] += r.excused
        a[3] += r.sz_mismatch
    tr = terminalreporter
    tr.write_sep("-", "code parity (elements, mismatched, excused, excused fraction, scale/zero mismatches)")
    rows = []
    for tid, (n, mis, exc, szm) in sorted(agg.items()):
        frac = exc / n if n else 0.0
        tr.write_line(f"{tid}: n={n} mismatched={mis} excused={exc} frac={frac:.2e} sz_mismatch={szm}")
        rows.append({"test": tid, "n": n, "mismatched": mis, "excused": exc, "excused_frac": frac,
                     "sz_mismatch": szm})
    out = os.environ.get("KVQ_PARITY_REPORT")
    if out:
        with open(out, "w") as f:
            json.dump(rows, f, indent=1)
