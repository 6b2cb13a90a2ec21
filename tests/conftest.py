import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Worst error of every recorded parity comparison, beside its tolerance."""
    parity = sys.modules.get("parity")
    if parity is None or not getattr(parity, "MARGINS", None):
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins (worst error / tolerance)")
    for case, what, err, tol in parity.MARGINS:
        tr.write_line(f"{case:<58} {what:<14} {err:10.3e} / {tol:.0e}  ({tol / max(err, 1e-300):8.1f}x)")
