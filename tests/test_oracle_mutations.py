"""The oracle's pins catch plausible mistakes: for each planted mistake of
tests/oracle_mutants.py the pins (tests/test_oracle_pins.py) run against the
mutated oracle in a child pytest, and at least one of them must fail.  The
children run side by side, one numpy thread each."""
import concurrent.futures as cf
import os
import subprocess
import sys

from tests.oracle_mutants import MUTANTS, ORACLE_SRC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_mutant_applies_once():
    src = open(ORACLE_SRC).read()
    for name, (old, _) in MUTANTS.items():
        assert src.count(old) == 1, name


def _run_pins(name: str, basetemp: str):
    env = dict(os.environ, RLT_ORACLE_MUTANT=name, OMP_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
         "-p", "tests.oracle_mutants", "-p", "no:cacheprovider", f"--basetemp={basetemp}"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout + r.stderr


def test_pins_catch_every_planted_mistake(tmp_path):
    names = sorted(MUTANTS)
    workers = max(1, min(len(names), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as ex:
        res = dict(zip(names, ex.map(lambda n: _run_pins(n, str(tmp_path / n)), names)))
    # exit code 1: the pins ran and one failed (2 would be a collection error)
    missed = {n: out[-1500:] for n, (rc, out) in res.items()
              if not (rc == 1 and "1 failed" in out)}
    assert not missed, f"mistakes no pin caught: {sorted(missed)}\n" + \
        "\n".join(f"--- {n}\n{o}" for n, o in missed.items())
