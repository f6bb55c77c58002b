import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def _has_cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_device():
    if not _has_cuda():
        pytest.skip("no CUDA device")
    import torch
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Print the worst parity ratios (|err| / bound) of the session, per output
    dtype and overall; with ESA_PARITY_REPORT=<path> also write them all as JSON."""
    mod = sys.modules.get("tests._parity")
    if mod is None:
        return
    worst = mod.worst_ratios()
    if not worst:
        return
    tr = terminalreporter
    tr.section("parity: worst |err| / bound")
    by_dtype = {}
    for (test, name), (r, dt) in worst.items():
        if r > by_dtype.get(dt, (0.0, None))[0]:
            by_dtype[dt] = (r, f"{test} {name}")
    for dt, (r, where) in sorted(by_dtype.items()):
        tr.write_line(f"{dt:>10}: {r:.3f}  ({where})")
    top = sorted(worst.items(), key=lambda kv: -kv[1][0])[:10]
    for (test, name), (r, dt) in top:
        tr.write_line(f"  {r:.3f}  {dt:>8}  {test}  {name}")
    path = os.environ.get("ESA_PARITY_REPORT")
    if path:
        import json
        rows = [{"test": t, "output": n, "ratio": r, "dtype": d} for (t, n), (r, d) in sorted(worst.items())]
        with open(path, "w") as f:
            json.dump(rows, f, indent=1)
