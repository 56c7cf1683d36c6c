"""The oracle's pins catch plausible mistakes: for each planted mistake of
tests/oracle_mutants.py the pins (tests/test_oracle_pins.py) run against the
mutated oracle in a child pytest and at least one of them must fail."""
import os
import subprocess
import sys

import pytest

from tests.oracle_mutants import MUTANTS, ORACLE_SRC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_mutant_applies_once():
    src = open(ORACLE_SRC).read()
    for name, (old, _) in MUTANTS.items():
        assert src.count(old) == 1, name


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    env = dict(os.environ, RLT_ORACLE_MUTANT=name)
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
         "-p", "tests.oracle_mutants", "-p", "no:cacheprovider",
         f"--basetemp={tmp_path / 'inner'}"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    out = r.stdout + r.stderr
    # exit code 1: tests ran and one failed (2 would be a collection error)
    assert r.returncode == 1 and "1 failed" in out, out[-3000:]
