import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: larger CPU-side oracle runs")


# A planted-mistake run (test_planted_mistakes.py) points the oracle at a build of
# a deliberately altered copy of its C source; the pins must then fail.
_MUTANT_LIB = os.environ.get("BLIN_ORACLE_MUTANT_LIB")
if _MUTANT_LIB:
    import oracle

    oracle.build = lambda force=False: _MUTANT_LIB
