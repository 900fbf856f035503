import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Selection near-ties per workload, as the parity rule requires them logged and counted."""
    from tests.msa_check import TIE_LOG
    if not TIE_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "selection near-ties (rows checked / rows differing / near-ties / cancellation near-ties)")
    for label in sorted(TIE_LOG):
        e = TIE_LOG[label]
        tr.write_line(f"{label}: {e['rows']} / {e['differing_rows']} / {e['near_ties']} / {e['cancel_ties']}")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True
