import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# tests/test_oracle_mutants.py runs the oracle pins against a mutated copy of the oracle
_MUTANT = os.environ.get("MOE_ORACLE_MUTANT_DIR")
if _MUTANT:
    sys.path.insert(0, _MUTANT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running on CPU")


@pytest.fixture(scope="session")
def oracle_lib():
    if _MUTANT:  # load the mutated copy by path, whatever sys.path says
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "oracle", os.path.join(_MUTANT, "oracle", "__init__.py"))
        mod = importlib.util.module_from_spec(spec)
        sys.modules["oracle"] = mod
        spec.loader.exec_module(mod)
    else:
        import oracle as mod
    mod.build()
    return mod
