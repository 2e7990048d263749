import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case")


if os.environ.get("MCS_ORACLE_MUTATION"):
    # a planted oracle mistake for tests/test_oracle_mutations.py (never set otherwise)
    import oracle_mutations

    oracle_mutations.apply(os.environ["MCS_ORACLE_MUTATION"])
