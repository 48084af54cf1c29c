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
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


# Achieved parity errors of the full-size workloads, printed in the terminal summary of every run (a
# passing test shows no output otherwise), so the margin under the tolerance is on record.
PARITY_RECORDS: list[tuple[str, float, float, float]] = []


GRAD_RECORDS: list[tuple[str, dict, float]] = []


@pytest.fixture(scope="session")
def parity_log():
    """Tests call parity_log(label, err_o, err_h, tol) to put an achieved error on record."""
    return lambda label, eo, eh, tol: PARITY_RECORDS.append((label, eo, eh, tol))


@pytest.fixture(scope="session")
def grad_log():
    """Backward tests call grad_log(label, {gradient: error}, tol) to put achieved errors on record."""
    return lambda label, errs, tol: GRAD_RECORDS.append((label, dict(errs), tol))


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not PARITY_RECORDS and not GRAD_RECORDS:
        return
    terminalreporter.section("achieved parity (max |gpu - oracle| / max |oracle|)")
    for label, eo, eh, tol in PARITY_RECORDS:
        terminalreporter.write_line(f"{label}: o {eo:.3e}  h_T {eh:.3e}  (tolerance {tol:.0e})")
    for label, errs, tol in GRAD_RECORDS:
        body = "  ".join(f"{k} {v:.2e}" for k, v in errs.items())
        terminalreporter.write_line(f"{label}: {body}  (tolerance {tol:.0e})")
