"""The oracle's pins catch plausible mistakes: each mutant in
tests/oracle_mutants.py is planted in a copy of oracle/dit_block.py (in a child
pytest process) and the pins of tests/test_oracle_pins.py and
tests/test_oracle_loop.py must then fail on an assertion. CPU only; the children run in parallel."""
import concurrent.futures as cf
import os
import subprocess
import sys

from tests.oracle_mutants import MUTANTS, VAE_MUTANTS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _pins_with(mutant: str, var: str = "H3_ORACLE_MUTANT",
               pins=("tests/test_oracle_pins.py", "tests/test_oracle_loop.py")):
    env = dict(os.environ, **{var: mutant})
    return subprocess.run(
        [sys.executable, "-m", "pytest", *pins, "-q", "-x", "-p", "no:cacheprovider",
         "-m", "not gpu"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def _check(results):
    # exit code 1: tests ran and some failed (2 or more would be a collection
    # or usage error, i.e. a broken mutant rather than a caught one)
    survived = [n for n, r in results.items() if r.returncode == 0]
    broken = {n: r.stdout[-400:] for n, r in results.items() if r.returncode not in (0, 1)}
    assert not broken, f"mutants that did not run: {broken}"
    assert not survived, f"mistakes no pin caught: {survived}"


def test_every_planted_vae_mistake_fails_a_pin():
    """The same for the VAE decoder oracle and tests/test_oracle_vae.py."""
    src = open(os.path.join(ROOT, "oracle", "vae_decoder.py")).read()
    for name, (old, _) in VAE_MUTANTS.items():
        assert old in src, f"mutant {name} no longer matches the oracle source"
    workers = max(1, min(8, os.cpu_count() or 1))
    run = lambda m: _pins_with(m, "H3_VAE_MUTANT", ("tests/test_oracle_vae.py",))
    with cf.ThreadPoolExecutor(workers) as ex:
        _check(dict(zip(VAE_MUTANTS, ex.map(run, VAE_MUTANTS))))


def test_every_planted_mistake_fails_a_pin():
    src = open(os.path.join(ROOT, "oracle", "dit_block.py")).read()
    for name, (old, _) in MUTANTS.items():
        assert old in src, f"mutant {name} no longer matches the oracle source"
    workers = max(1, min(8, os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as ex:
        results = dict(zip(MUTANTS, ex.map(_pins_with, MUTANTS)))
    # exit code 1: tests ran and some failed (2 or more would be a collection
    # or usage error, i.e. a broken mutant rather than a caught one)
    survived = [n for n, r in results.items() if r.returncode == 0]
    broken = {n: r.stdout[-400:] for n, r in results.items() if r.returncode not in (0, 1)}
    assert not broken, f"mutants that did not run: {broken}"
    assert not survived, f"mistakes no pin caught: {survived}"
