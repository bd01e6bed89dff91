import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_native():
    """Build the CUDA library and the device generator in-tree when stale (nvcc cross-compiles)."""
    import importlib.util

    import synth.device as sd

    # build.py is loaded by path: importing the package itself needs the built library.
    spec = importlib.util.spec_from_file_location(
        "_hisa_build", os.path.join(ROOT, "hierarchical_sparse_attention_block_b200", "build.py"))
    hb = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(hb)
    hb.build()
    sd.build()


def pytest_configure(config):
    _build_native()
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    return oracle.Oracle()
