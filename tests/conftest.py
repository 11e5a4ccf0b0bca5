import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libaxr.so")


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device on this machine")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def axr_lib():
    """The CUDA library, built in-tree if missing (nvcc cross-compiles without a GPU)."""
    from lut_attention_b200 import axr, build

    if not os.path.exists(axr.LIB_PATH):
        build.build()
    return axr.library()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Full-size parity counts (tests/full_parity.py), one line per workload, at
    the end of the run's output."""
    mod = sys.modules.get("full_parity")
    if mod is not None and mod.REPORTS:
        terminalreporter.write_sep("-", "full-size parity with the oracle (boundary window 1e-6)")
        for line in mod.REPORTS:
            terminalreporter.write_line(line)
