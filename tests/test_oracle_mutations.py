"""Each planted oracle mistake (tests/oracle_mutations.py: an uncentered PDDP, a ceil(m/2)
split, a flipped sign rule, a missing LSE, ties to the higher key, unsorted indices) makes at
least one of the oracle's pins in tests/test_oracle.py fail, and the unmodified oracle passes
them all (CPU only)."""

import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
from oracle_mutations import MUTATIONS  # noqa: E402


def _run_pins(mutation):
    env = dict(os.environ)
    env.pop("MCS_ORACLE_MUTATION", None)
    if mutation:
        env["MCS_ORACLE_MUTATION"] = mutation
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle.py"), "-q", "-x",
                           "-p", "no:cacheprovider"], cwd=os.path.dirname(HERE), env=env, capture_output=True,
                          text=True, timeout=600)


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation):
    r = _run_pins(mutation)
    assert r.returncode != 0, f"no pin caught {mutation}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout


def test_unmodified_oracle_passes_its_pins():
    r = _run_pins(None)
    assert r.returncode == 0, r.stdout[-2000:]
