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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the parity reports the GPU tests recorded: tokens compared, near-tie tokens
    exempted from the routing check, max-abs and relative L2 error against the oracle."""
    try:
        from tests import parity
    except ImportError:  # pragma: no cover
        return
    if not parity.REPORTS:
        return
    tr = terminalreporter
    tr.write_line("parity against the oracle (tokens compared, exempt near-ties, max-abs, "
                  "rel-L2):")
    for name, r in parity.REPORTS:
        tr.write_line(f"  {name}: tokens={r.get('tokens')} exempt={r.get('exempt')} "
                      f"max_abs={r.get('max_abs', float('nan')):.3g} "
                      f"rel_l2={r.get('rel_l2', float('nan')):.3g} ok={r.get('ok')}")
