import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of CPU oracle time")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


def _build_library(checked: bool = False):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "efla_build", os.path.join(ROOT, "delta_rule_linear_02_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build(checked=checked)


@pytest.fixture(scope="session")
def efla():
    """The library binding (builds libefla.so in-tree first if it is missing or stale)."""
    _build_library()
    import delta_rule_linear_02_b200 as m
    return m


@pytest.fixture(scope="session")
def cuda(efla):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    torch.backends.cuda.matmul.allow_tf32 = False
    return torch.device("cuda", 0)


@pytest.fixture
def efla_checked(efla, cuda):
    """The binding with its `lib` swapped for the checked build (libefla_checked.so) for the
    duration of one test."""
    _build_library(checked=True)
    saved = efla.lib
    efla.lib = efla.load_checked()
    try:
        yield efla
    finally:
        efla.lib = saved
