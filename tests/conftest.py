import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# With H3_ORACLE_MUTANT set (only tests/test_oracle_mutations.py sets it, in a
# child process), the oracle module is replaced by a copy with one planted
# mistake from tests/oracle_mutants.py, so that the pins can be shown to catch it.
_MUTANT = os.environ.get("H3_ORACLE_MUTANT")
if _MUTANT:
    import types

    import oracle
    from tests.oracle_mutants import MUTANTS

    _old, _new = MUTANTS[_MUTANT]
    _path = os.path.join(ROOT, "oracle", "dit_block.py")
    with open(_path) as _fh:
        _src = _fh.read()
    assert _old in _src, _MUTANT
    _mod = types.ModuleType("oracle.dit_block")
    _mod.__file__ = _path
    sys.modules["oracle.dit_block"] = _mod
    exec(compile(_src.replace(_old, _new, 1), _path, "exec"), _mod.__dict__)
    oracle.dit_block = _mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
