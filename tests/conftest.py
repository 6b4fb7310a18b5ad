import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# With H3_ORACLE_MUTANT set (only tests/test_oracle_mutations.py sets it, in a
# child process), the oracle module is replaced by a copy with one planted
# mistake from tests/oracle_mutants.py, so that the pins can be shown to catch it.
# H3_VAE_MUTANT does the same for oracle/vae_decoder.py.
def _plant(module: str, table: dict, name: str) -> None:
    import types

    import oracle

    _old, _new = table[name]
    path = os.path.join(ROOT, "oracle", module + ".py")
    with open(path) as fh:
        src = fh.read()
    assert _old in src, name
    mod = types.ModuleType("oracle." + module)
    mod.__file__ = path
    sys.modules["oracle." + module] = mod
    exec(compile(src.replace(_old, _new, 1), path, "exec"), mod.__dict__)
    setattr(oracle, module, mod)


if os.environ.get("H3_ORACLE_MUTANT"):
    from tests.oracle_mutants import MUTANTS

    _plant("dit_block", MUTANTS, os.environ["H3_ORACLE_MUTANT"])
if os.environ.get("H3_VAE_MUTANT"):
    from tests.oracle_mutants import VAE_MUTANTS

    _plant("vae_decoder", VAE_MUTANTS, os.environ["H3_VAE_MUTANT"])


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
