"""Each planted mistake in the oracle (a build with ORACLE_MUTANT=n, on the CPU) must
make at least one pin in test_oracle_pins.py fail: the pins are sensitive to a
readout from the wrong state, a dropped decay, a dropped input gate, a wrong-state dq,
a sign error in dg, a missing gate in dv, and an undecayed state gradient."""
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7])
def test_planted_mistake_is_caught(mutant, tmp_path):
    lib = oracle_build.build_mutant(mutant, str(tmp_path))
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {mutant} passed every pin:\n{r.stdout[-2000:]}"
