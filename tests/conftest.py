import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


@pytest.fixture(scope="session")
def gdn():
    """The CUDA library's Python binding, loaded on a GPU machine only."""
    if not gpu_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_77_b200 as gdn_mod
    gdn_mod.load()  # raises if the native library is missing: no fallback
    return gdn_mod


@pytest.fixture(scope="session")
def oracle_threads():
    return int(os.environ.get("GDN_ORACLE_THREADS", "0")) or None
