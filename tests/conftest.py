import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    from oracle import oracle as O
    O.build()
    return O


@pytest.fixture(autouse=True)
def _parity_label(request):
    """Tag every oracle comparison made by this test with its id (oracle.PARITY_LOG)."""
    from oracle import oracle as O
    O.PARITY_LABEL[0] = request.node.nodeid
    yield
    O.PARITY_LABEL[0] = ""


def pytest_terminal_summary(terminalreporter):
    """Per test: the worst normwise relative error (what the tolerances bound) and the worst
    elementwise p99 relative error (floor 1e-6 max|ref|) of its comparisons against the oracle.
    HMD_PARITY_LOG=<path> also writes every comparison there as JSON."""
    O = sys.modules.get("oracle.oracle")
    if O is None or not O.PARITY_LOG:
        return
    worst = {}
    for e in O.PARITY_LOG:
        w = worst.setdefault(e["test"] or "(outside a test)", [0.0, 0.0, 0])
        w[0] = max(w[0], e["normwise"])
        w[1] = max(w[1], e["p99_elementwise"])
        w[2] += 1
    tr = terminalreporter
    tr.write_sep("-", f"parity against the oracle: {len(O.PARITY_LOG)} comparisons")
    tr.write_line(f"{'normwise':>10} {'p99 elem':>10} {'n':>4}  test")
    for name, (nw, p99, n) in sorted(worst.items(), key=lambda kv: -kv[1][1])[:40]:
        tr.write_line(f"{nw:10.3e} {p99:10.3e} {n:4d}  {name}")
    nw = max(v[0] for v in worst.values())
    p99 = max(v[1] for v in worst.values())
    tr.write_line(f"worst normwise {nw:.3e}, worst elementwise p99 {p99:.3e}")
    path = os.environ.get("HMD_PARITY_LOG")
    if path:
        with open(path, "w") as f:
            json.dump(O.PARITY_LOG, f)
