"""Every planted oracle slip must make the pin suite fail (CPU only)."""
import os
import subprocess
import sys

import pytest

from oracle_mutants import MUTANT_NAMES

HERE = os.path.dirname(os.path.abspath(__file__))


def _run_pins(mutant):
    env = dict(os.environ, SFX_ORACLE_MUTANT=mutant)
    return subprocess.run(
        [sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"),
         "-q", "-x", "-p", "no:cacheprovider"],
        cwd=os.path.dirname(HERE), env=env, capture_output=True, text=True, timeout=300)


def test_unmutated_pins_pass():
    r = _run_pins("")
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", MUTANT_NAMES)
def test_mutant_is_caught(mutant):
    r = _run_pins(mutant)
    assert r.returncode != 0, f"mutant {mutant} passed every pin:\n{r.stdout[-1500:]}"
