import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload; minutes of CPU oracle time")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library, loaded through the Python binding (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_tok_b200 import sparstar
    return sparstar.load()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print, per checked configuration, how many mask rows and output blocks were compared."""
    try:
        from tests.parity import LOG
    except Exception:  # the parity module was never imported (CPU-only run)
        return
    if LOG:
        terminalreporter.write_line("parity coverage (GPU vs oracle):")
        for line in LOG:
            terminalreporter.write_line("  " + line)
