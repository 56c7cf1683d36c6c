import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


@pytest.hookimpl(tryfirst=True)
def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    # the tests' temporary files stay inside the repository
    if not config.option.basetemp:
        config.option.basetemp = os.path.join(ROOT, ".pytest_tmp")


def build_library():
    """Compile librlt.so if a source changed (loads build.py by path, so the
    package -- which loads the library -- is not imported first)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "rlt_build", os.path.join(ROOT, "stateful_decoding_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()
