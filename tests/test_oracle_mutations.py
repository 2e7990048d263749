"""Each planted oracle mistake (tests/oracle_mutations.py: an uncentered PDDP, a ceil(m/2)
split, a flipped sign rule, a missing LSE, ties to the higher key, unsorted indices; in the
selection variants a block max instead of the block mass, BSA pooling by the first key, a
per-query softmax not renormalised over its keys) makes at least one of the oracle's pins
fail, and the unmodified oracle passes them all (CPU only)."""

import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
from oracle_mutations import MUTATIONS, PINS  # noqa: E402


def _run_pins(mutation, module="test_oracle.py"):
    env = dict(os.environ)
    env.pop("MCS_ORACLE_MUTATION", None)
    if mutation:
        env["MCS_ORACLE_MUTATION"] = mutation
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, module), "-q", "-x",
                           "-p", "no:cacheprovider"], cwd=os.path.dirname(HERE), env=env, capture_output=True,
                          text=True, timeout=600)


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation):
    r = _run_pins(mutation, PINS[mutation])
    assert r.returncode != 0, f"no pin caught {mutation}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout


@pytest.mark.parametrize("module", ["test_oracle.py", "test_oracle_variants.py"])
def test_unmodified_oracle_passes_its_pins(module):
    r = _run_pins(None, module)
    assert r.returncode == 0, r.stdout[-2000:]
