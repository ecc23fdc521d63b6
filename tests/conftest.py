import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def gpu_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


@pytest.fixture(scope="session")
def lib():
    """The CUDA library binding; a GPU test fails loudly if it cannot load."""
    import exact_tiled_attention_38_b200 as eta

    eta.load_library()
    return eta


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print every GPU-vs-oracle comparison of the session: its max errors and
    how many outputs passed under the one-ulp allowance of `parity.py`."""
    try:
        import parity
    except Exception:  # pragma: no cover
        return
    lines = parity.summary_lines()
    if not lines:
        return
    n_allow = sum(r["n_ulp_allowance"] for _, r in parity.RECORDS)
    terminalreporter.section(f"parity against the fp64 oracle ({len(lines)} comparisons, "
                             f"{n_allow} outputs under the one-ulp allowance)")
    for line in lines:
        terminalreporter.write_line(line)
