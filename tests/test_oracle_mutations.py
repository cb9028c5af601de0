"""Each planted mistake in the oracle (tests/oracle_mutations.py, applied on the CPU in a child
pytest run) must make some pin fail: the layer's mistakes in tests/test_oracle_pins.py, those of
the fused QKV stage, awq_w4a16 and the MLP pair in their own pin files."""
import os
import subprocess
import sys

import pytest

from tests.oracle_mutations import MUTATIONS, PIN_FILES

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("name", MUTATIONS + sorted(PIN_FILES))
def test_pins_catch_planted_mistake(name):
    env = dict(os.environ, SVDQ_ORACLE_MUTATION=name)
    pins = PIN_FILES.get(name, "tests/test_oracle_pins.py")
    r = subprocess.run([sys.executable, "-m", "pytest", pins, "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"{name}: pins passed or errored\n{r.stdout[-2000:]}\n{r.stderr[-2000:]}"
    assert " failed" in r.stdout, r.stdout[-2000:]
