"""Each planted mistake in the oracle (tests/oracle_mutations.py, applied on the CPU in a child
pytest run) must make some pin in tests/test_oracle_pins.py fail."""
import os
import subprocess
import sys

import pytest

from tests.oracle_mutations import MUTATIONS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("name", MUTATIONS)
def test_pins_catch_planted_mistake(name):
    env = dict(os.environ, SVDQ_ORACLE_MUTATION=name)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"{name}: pins passed or errored\n{r.stdout[-2000:]}\n{r.stderr[-2000:]}"
    assert " failed" in r.stdout, r.stdout[-2000:]
